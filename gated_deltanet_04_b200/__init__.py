"""Python binding of libgdn: the gated delta rule on B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in libgdn's
CUDA kernels; this module checks tensor shapes/dtypes, allocates outputs with
torch (device memory is the only thing torch is used for), and passes raw
device pointers plus the current CUDA stream to the C ABI declared in
include/gdn.h.  There is no CPU path: if libgdn.so is missing or no CUDA device
is present, the calls raise.

Entry points (same names as the C ABI):
    gdn_prefill(q, k, v, g, beta, initial_state=None, cu_seqlens=None, ...)
    gdn_decode_step(q, k, v, g, beta, state, ...)
    gdn_decode_step_bf16_state(q, k, v, g, beta, state, ...)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["gdn_prefill", "gdn_decode_step", "gdn_decode_step_bf16_state", "gdn_decode_step_slots",
           "gdn_short_conv_norm", "gdn_prefill_conv", "gdn_prefill_conv_workspace_bytes",
           "gdn_prefill_host", "gdn_prefill_host_scratch_bytes", "gdn_prefill_slots",
           "gdn_prefill_workspace_bytes", "library",
           "GdnError", "LIB_PATH", "STATUS", "KERNELS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn.so")

STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARGUMENT", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_CUDA",
          4: "GDN_ERR_TIMEOUT", 5: "GDN_ERR_BAD_SEQLENS", 6: "GDN_ERR_BAD_SLOT", 7: "GDN_ERR_RANGE"}
DTYPE = {torch.bfloat16: 0, torch.float32: 1}
# gdn_order values of include/gdn.h: where the recall S k is taken
ORDERS = {"standard": 0, "recall_first": 1}
# gdn_prefill_kernel values of include/gdn.h
KERNELS = {"auto": 0, "cluster": 1, "single_cta": 2, "recurrent": 3, "pool": 4}

_lib = None
_lock = threading.Lock()


class GdnError(RuntimeError):
    def __init__(self, code, where):
        self.code = int(code)
        super().__init__(f"{where} failed: {STATUS.get(self.code, self.code)}")


def library():
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libgdn.so not built at {LIB_PATH}; run "
                                  "`python -m gated_deltanet_04_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
            lib.gdn_prefill.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32,
                                        i32, i32, i32, vp, vp, vp, sz, vp, vp]
            lib.gdn_prefill.restype = ctypes.c_int
            lib.gdn_prefill_ex.argtypes = lib.gdn_prefill.argtypes + [ctypes.c_int]
            lib.gdn_prefill_ex.restype = ctypes.c_int
            lib.gdn_decode_step.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, i32, i32, i32, i32,
                                            i32, vp, vp, vp]
            lib.gdn_decode_step.restype = ctypes.c_int
            lib.gdn_decode_step_bf16_state.argtypes = lib.gdn_decode_step.argtypes
            lib.gdn_decode_step_bf16_state.restype = ctypes.c_int
            lib.gdn_prefill_order.argtypes = lib.gdn_prefill_ex.argtypes + [ctypes.c_int]
            lib.gdn_prefill_order.restype = ctypes.c_int
            lib.gdn_decode_step_order.argtypes = lib.gdn_decode_step.argtypes + [ctypes.c_int]
            lib.gdn_decode_step_order.restype = ctypes.c_int
            lib.gdn_decode_step_slots.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, i32, vp, vp,
                                                  i32, i32, i32, i32, i32, vp, vp, vp]
            lib.gdn_decode_step_slots.restype = ctypes.c_int
            lib.gdn_short_conv_norm.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, vp,
                                                i32, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp]
            lib.gdn_short_conv_norm.restype = ctypes.c_int
            lib.gdn_prefill_conv.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp, i32, i64, i32, i32, i32, i32, i32, vp, vp,
                                             vp, sz, vp, vp]
            lib.gdn_prefill_conv.restype = ctypes.c_int
            lib.gdn_prefill_conv_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32]
            lib.gdn_prefill_conv_workspace_bytes.restype = sz
            lib.gdn_prefill_slots.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, i32, vp, vp,
                                              vp, i32, i64, i32, i32, i32, i32, i32, vp, vp, sz,
                                              vp, vp]
            lib.gdn_prefill_slots.restype = ctypes.c_int
            lib.gdn_prefill_slots_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32, i32]
            lib.gdn_prefill_slots_workspace_bytes.restype = sz
            lib.gdn_prefill_host.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, i64, i32, i32,
                                             i32, i32, i32, vp, vp, i64, vp, sz, vp, vp]
            lib.gdn_prefill_host.restype = ctypes.c_int
            lib.gdn_prefill_host_scratch_bytes.argtypes = [i64, i32, i32, i32, i32, i32,
                                                           ctypes.c_int, i64]
            lib.gdn_prefill_host_scratch_bytes.restype = sz
            lib.gdn_prefill_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32, i32]
            lib.gdn_prefill_workspace_bytes.restype = sz
            lib.gdn_prefill_ex_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32, i32,
                                                           ctypes.c_int]
            lib.gdn_prefill_ex_workspace_bytes.restype = sz
            lib.gdn_status_string.argtypes = [ctypes.c_int]
            lib.gdn_status_string.restype = ctypes.c_char_p
            lib.gdn_version.argtypes = []
            lib.gdn_version.restype = i32
            _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(t, name, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_prefill_conv_workspace_bytes(N, T, Hqk, Hv, Dk, Dv):
    """Scratch bytes gdn_prefill_conv needs (0: none, or unsupported shapes)."""
    return int(library().gdn_prefill_conv_workspace_bytes(N, T, Hqk, Hv, Dk, Dv))


def gdn_prefill_host_scratch_bytes(T, Hqk, Hv, Dk, Dv, chunk=0, dtype=torch.bfloat16,
                                   segment_tokens=0):
    """Device scratch bytes gdn_prefill_host needs."""
    return int(library().gdn_prefill_host_scratch_bytes(T, Hqk, Hv, Dk, Dv, chunk, DTYPE[dtype],
                                                        segment_tokens))


def gdn_prefill_host(q, k, v, g, beta, initial_state=None, *, o=None, final_state=None,
                     output_final_state=True, chunk=0, segment_tokens=0, scratch=None,
                     error_flag=None, device=None, stream=None):
    """One sequence's prefill from HOST tensors (the C entry point
    gdn_prefill_host): q, k [T,Hqk,Dk], v [T,Hv,Dv], g, beta [T,Hv], optional
    initial_state [Hv,Dv,Dk], all on the CPU (pinned for overlapped copies).
    The sequence streams through the device in segments.  Returns (o,
    final_state) as CPU tensors; the copies into them are complete when
    `stream` (default: the current stream of `device`) has reached them."""
    lib = library()
    cpu = torch.device("cpu")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    _check(q, "q", (T, Hqk, Dk), q.dtype, cpu)
    _check(k, "k", (T, Hqk, Dk), q.dtype, cpu)
    _check(v, "v", (T, Hv, Dv), q.dtype, cpu)
    _check(g, "g", (T, Hv), torch.float32, cpu)
    _check(beta, "beta", (T, Hv), torch.float32, cpu)
    if initial_state is not None:
        _check(initial_state, "initial_state", (Hv, Dv, Dk), torch.float32, cpu)
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=q.dtype).pin_memory()
    _check(o, "o", (T, Hv, Dv), q.dtype, cpu)
    if final_state is None and output_final_state:
        final_state = torch.empty((Hv, Dv, Dk), dtype=torch.float32).pin_memory()
    if final_state is not None:
        _check(final_state, "final_state", (Hv, Dv, Dk), torch.float32, cpu)
    need = int(lib.gdn_prefill_host_scratch_bytes(T, Hqk, Hv, Dk, Dv, chunk, DTYPE[q.dtype],
                                                  segment_tokens))
    if scratch is None:
        scratch = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if error_flag is not None:
        _check(error_flag, "error_flag", tuple(error_flag.shape), torch.int32, dev)
    st = torch.cuda.current_stream(dev) if stream is None else stream
    rc = lib.gdn_prefill_host(_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g), _ptr(beta),
                              _ptr(initial_state), T, Hqk, Hv, Dk, Dv, chunk, _ptr(o),
                              _ptr(final_state), segment_tokens, _ptr(scratch),
                              scratch.numel() * scratch.element_size(), _ptr(error_flag),
                              ctypes.c_void_p(st.cuda_stream))
    if rc != 0:
        raise GdnError(rc, "gdn_prefill_host")
    return o, final_state


def gdn_prefill_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk=0, kernel="auto"):
    return int(library().gdn_prefill_ex_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk,
                                                        KERNELS[kernel]))


def gdn_prefill(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, chunk=0, o=None,
                final_state=None, output_final_state=True, workspace=None, error_flag=None,
                stream=None, kernel="auto", order="standard"):
    """Chunk-parallel prefill of the gated delta rule on the GPU.

    q, k [T,Hqk,Dk] and v [T,Hv,Dv] (bf16 or fp32, same dtype); g, beta [T,Hv] fp32;
    initial_state [N,Hv,Dv,Dk] fp32 or None; cu_seqlens int32 [N+1] on the device or None.
    Returns (o [T,Hv,Dv], final_state [N,Hv,Dv,Dk] or None).  ``final_state`` may be
    ``initial_state`` for an in-place update.  Asynchronous on the current stream.
    ``kernel``: "auto", "pool", "cluster", "single_cta" or "recurrent" (see gdn_prefill_ex).
    ``order``: "standard", or "recall_first" (the recall S k before the decay; the C
    entry point gdn_prefill_order).
    """
    lib = library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_prefill runs on CUDA tensors only")
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    _check(k, "k", (T, Hqk, Dk), q.dtype, dev)
    _check(q, "q", (T, Hqk, Dk), q.dtype, dev)
    _check(v, "v", (T, Hv, Dv), q.dtype, dev)
    _check(g, "g", (T, Hv), torch.float32, dev)
    _check(beta, "beta", (T, Hv), torch.float32, dev)
    if cu_seqlens is None:
        N = 1
    else:
        N = cu_seqlens.shape[0] - 1
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, Hv, Dv, Dk), torch.float32, dev)
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=q.dtype, device=dev)
    _check(o, "o", (T, Hv, Dv), q.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, Hv, Dv, Dk), dtype=torch.float32, device=dev)
    if final_state is not None:
        _check(final_state, "final_state", (N, Hv, Dv, Dk), torch.float32, dev)
    ws_bytes = 0
    if workspace is not None:
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        need = int(lib.gdn_prefill_ex_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk, KERNELS[kernel]))
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            ws_bytes = need
    args = (_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), N, T, Hqk, Hv, Dk, Dv, chunk, _ptr(o), _ptr(final_state),
            _ptr(workspace), ws_bytes, _ptr(error_flag), _stream(stream), KERNELS[kernel])
    if order == "standard":
        rc = lib.gdn_prefill_ex(*args)
    else:
        rc = lib.gdn_prefill_order(*args, ORDERS[order])
    if rc != 0:
        raise GdnError(rc, "gdn_prefill")
    return o, final_state


def gdn_decode_step(q, k, v, g, beta, state, *, o=None, error_flag=None, stream=None,
                    order="standard"):
    """One-token update of N sequences, in place on ``state`` [N,Hv,Dv,Dk] fp32.

    q, k [N,Hqk,Dk], v [N,Hv,Dv] (bf16 or fp32); g, beta [N,Hv] fp32.  Returns o [N,Hv,Dv].
    ``order``: "standard" or "recall_first" (the C entry point gdn_decode_step_order).
    """
    lib = library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_decode_step runs on CUDA tensors only")
    N, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    _check(k, "k", (N, Hqk, Dk), q.dtype, dev)
    _check(v, "v", (N, Hv, Dv), q.dtype, dev)
    _check(g, "g", (N, Hv), torch.float32, dev)
    _check(beta, "beta", (N, Hv), torch.float32, dev)
    _check(state, "state", (N, Hv, Dv, Dk), torch.float32, dev)
    if o is None:
        o = torch.empty((N, Hv, Dv), dtype=q.dtype, device=dev)
    _check(o, "o", (N, Hv, Dv), q.dtype, dev)
    args = (_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g), _ptr(beta), _ptr(state), N, Hqk,
            Hv, Dk, Dv, _ptr(o), _ptr(error_flag), _stream(stream))
    if order == "standard":
        rc = lib.gdn_decode_step(*args)
    else:
        rc = lib.gdn_decode_step_order(*args, ORDERS[order])
    if rc != 0:
        raise GdnError(rc, "gdn_decode_step")
    return o


def gdn_decode_step_slots(q, k, v, g, beta, state_pool, slot_idx, reset=None, *, o=None,
                          error_flag=None, stream=None):
    """One decode step for continuous batching: entry n's state is
    ``state_pool[slot_idx[n]]`` ([num_slots,Hv,Dv,Dk] fp32, updated in place);
    ``reset`` (int32 [N] or None) marks entries that start from a zero state.
    ``slot_idx`` is int32 [N] on the device, distinct values in [0, num_slots).
    q, k [N,Hqk,Dk], v [N,Hv,Dv] (bf16 or fp32); g, beta [N,Hv] fp32.  Returns o."""
    lib = library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_decode_step_slots runs on CUDA tensors only")
    N, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    S = state_pool.shape[0]
    _check(k, "k", (N, Hqk, Dk), q.dtype, dev)
    _check(v, "v", (N, Hv, Dv), q.dtype, dev)
    _check(g, "g", (N, Hv), torch.float32, dev)
    _check(beta, "beta", (N, Hv), torch.float32, dev)
    _check(state_pool, "state_pool", (S, Hv, Dv, Dk), torch.float32, dev)
    _check(slot_idx, "slot_idx", (N,), torch.int32, dev)
    if reset is not None:
        _check(reset, "reset", (N,), torch.int32, dev)
    if o is None:
        o = torch.empty((N, Hv, Dv), dtype=q.dtype, device=dev)
    _check(o, "o", (N, Hv, Dv), q.dtype, dev)
    rc = lib.gdn_decode_step_slots(_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g), _ptr(beta),
                                   _ptr(state_pool), S, _ptr(slot_idx), _ptr(reset), N, Hqk, Hv,
                                   Dk, Dv, _ptr(o), _ptr(error_flag), _stream(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_decode_step_slots")
    return o


def gdn_prefill_slots(q, k, v, g, beta, state_pool, slot_idx, reset=None, cu_seqlens=None, *,
                      chunk=0, o=None, workspace=None, error_flag=None, stream=None):
    """Prefill for continuous batching: sequence n starts from
    ``state_pool[slot_idx[n]]`` ([num_slots,Hv,Dv,Dk] fp32, updated in place),
    or from zeros when ``reset[n]`` is nonzero, and its final state goes back
    to that slot.  q, k [T,Hqk,Dk], v [T,Hv,Dv], g, beta [T,Hv] as gdn_prefill;
    slot_idx (and reset) int32 [N] on the device; cu_seqlens int32 [N+1] or
    None (N = 1).  Returns o."""
    lib = library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_prefill_slots runs on CUDA tensors only")
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    N = 1 if cu_seqlens is None else cu_seqlens.shape[0] - 1
    S = state_pool.shape[0]
    _check(k, "k", (T, Hqk, Dk), q.dtype, dev)
    _check(v, "v", (T, Hv, Dv), q.dtype, dev)
    _check(g, "g", (T, Hv), torch.float32, dev)
    _check(beta, "beta", (T, Hv), torch.float32, dev)
    _check(state_pool, "state_pool", (S, Hv, Dv, Dk), torch.float32, dev)
    _check(slot_idx, "slot_idx", (N,), torch.int32, dev)
    if reset is not None:
        _check(reset, "reset", (N,), torch.int32, dev)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=q.dtype, device=dev)
    _check(o, "o", (T, Hv, Dv), q.dtype, dev)
    need = int(lib.gdn_prefill_slots_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    rc = lib.gdn_prefill_slots(_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g), _ptr(beta),
                               _ptr(state_pool), S, _ptr(slot_idx), _ptr(reset), _ptr(cu_seqlens),
                               N, T, Hqk, Hv, Dk, Dv, chunk, _ptr(o), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _ptr(error_flag),
                               _stream(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_prefill_slots")
    return o


def gdn_short_conv_norm(xq, xk, xv, wq, wk, wv, cu_seqlens=None, conv_state=None, *,
                        conv_state_out=None, output_conv_state=False, error_flag=None,
                        stream=None):
    """The mixer's kernel-4 causal convolution on the q, k, v channels, then q, k
    normalised per head: returns (q, k, v[, conv_state_out]) ready for gdn_prefill.

    xq, xk [T,Hqk,128], xv [T,Hv,128] (bf16 or fp32); wq, wk [Hqk*128,4], wv
    [Hv*128,4] fp32; cu_seqlens int32 [N+1] or None; conv_state [N,3,C] fp32 or
    None with C = 2*Hqk*128 + Hv*128 (q, k, v channels).  With
    output_conv_state (or a conv_state_out tensor, which may be conv_state) the
    new conv state is returned too."""
    lib = library()
    dev = xq.device
    if dev.type != "cuda":
        raise ValueError("gdn_short_conv_norm runs on CUDA tensors only")
    T, Hqk, Dk = xq.shape
    Hv, Dv = xv.shape[1], xv.shape[2]
    if xq.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {xq.dtype}")
    _check(xk, "xk", (T, Hqk, Dk), xq.dtype, dev)
    _check(xv, "xv", (T, Hv, Dv), xq.dtype, dev)
    _check(wq, "wq", (Hqk * Dk, 4), torch.float32, dev)
    _check(wk, "wk", (Hqk * Dk, 4), torch.float32, dev)
    _check(wv, "wv", (Hv * Dv, 4), torch.float32, dev)
    if cu_seqlens is None:
        N = 1
    else:
        N = cu_seqlens.shape[0] - 1
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    C = 2 * Hqk * Dk + Hv * Dv
    if conv_state is not None:
        _check(conv_state, "conv_state", (N, 3, C), torch.float32, dev)
    if conv_state_out is None and output_conv_state:
        conv_state_out = torch.empty((N, 3, C), dtype=torch.float32, device=dev)
    if conv_state_out is not None:
        _check(conv_state_out, "conv_state_out", (N, 3, C), torch.float32, dev)
    q = torch.empty_like(xq)
    k = torch.empty_like(xk)
    v = torch.empty_like(xv)
    rc = lib.gdn_short_conv_norm(_ptr(xq), _ptr(xk), _ptr(xv), DTYPE[xq.dtype], _ptr(wq), _ptr(wk),
                                 _ptr(wv), _ptr(conv_state), _ptr(conv_state_out),
                                 _ptr(cu_seqlens), N, T, Hqk, Hv, Dk, Dv, _ptr(q), _ptr(k),
                                 _ptr(v), _ptr(error_flag), _stream(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_short_conv_norm")
    return (q, k, v, conv_state_out) if conv_state_out is not None else (q, k, v)


def gdn_decode_step_bf16_state(q, k, v, g, beta, state, *, o=None, error_flag=None, stream=None):
    """gdn_decode_step for a state stored in bfloat16: ``state`` [N,Hv,128,128]
    bfloat16, updated in place (computed in fp32, rounded to nearest even).
    q, k [N,Hqk,128], v [N,Hv,128] (bf16 or fp32); g, beta [N,Hv] fp32.
    Returns o [N,Hv,128]."""
    lib = library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_decode_step_bf16_state runs on CUDA tensors only")
    N, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if q.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {q.dtype}")
    _check(k, "k", (N, Hqk, Dk), q.dtype, dev)
    _check(v, "v", (N, Hv, Dv), q.dtype, dev)
    _check(g, "g", (N, Hv), torch.float32, dev)
    _check(beta, "beta", (N, Hv), torch.float32, dev)
    _check(state, "state", (N, Hv, Dv, Dk), torch.bfloat16, dev)
    if o is None:
        o = torch.empty((N, Hv, Dv), dtype=q.dtype, device=dev)
    _check(o, "o", (N, Hv, Dv), q.dtype, dev)
    rc = lib.gdn_decode_step_bf16_state(_ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(g),
                                        _ptr(beta), _ptr(state), N, Hqk, Hv, Dk, Dv, _ptr(o),
                                        _ptr(error_flag), _stream(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_decode_step_bf16_state")
    return o


def gdn_prefill_conv(xq, xk, xv, wq, wk, wv, g, beta, initial_state=None, cu_seqlens=None,
                     conv_state=None, *, conv_state_out=None, output_conv_state=False, o=None,
                     final_state=None, output_final_state=True, workspace=None, error_flag=None,
                     stream=None):
    """gdn_short_conv_norm followed by gdn_prefill in one call, with the front end
    fused into the pool prefill kernel's load stage (the C entry point
    gdn_prefill_conv).  Arguments as the two calls: raw channel inputs xq, xk
    [T,Hqk,128], xv [T,Hv,128] bf16, filters, conv state, then the prefill's.
    Returns (o, final_state[, conv_state_out])."""
    lib = library()
    dev = xq.device
    if dev.type != "cuda":
        raise ValueError("gdn_prefill_conv runs on CUDA tensors only")
    T, Hqk, Dk = xq.shape
    Hv, Dv = xv.shape[1], xv.shape[2]
    if xq.dtype not in DTYPE:
        raise ValueError(f"unsupported io dtype {xq.dtype}")
    _check(xk, "xk", (T, Hqk, Dk), xq.dtype, dev)
    _check(xv, "xv", (T, Hv, Dv), xq.dtype, dev)
    _check(wq, "wq", (Hqk * Dk, 4), torch.float32, dev)
    _check(wk, "wk", (Hqk * Dk, 4), torch.float32, dev)
    _check(wv, "wv", (Hv * Dv, 4), torch.float32, dev)
    _check(g, "g", (T, Hv), torch.float32, dev)
    _check(beta, "beta", (T, Hv), torch.float32, dev)
    if cu_seqlens is None:
        N = 1
    else:
        N = cu_seqlens.shape[0] - 1
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    C = 2 * Hqk * Dk + Hv * Dv
    if conv_state is not None:
        _check(conv_state, "conv_state", (N, 3, C), torch.float32, dev)
    if conv_state_out is None and output_conv_state:
        conv_state_out = torch.empty((N, 3, C), dtype=torch.float32, device=dev)
    if conv_state_out is not None:
        _check(conv_state_out, "conv_state_out", (N, 3, C), torch.float32, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, Hv, Dv, Dk), torch.float32, dev)
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=xq.dtype, device=dev)
    _check(o, "o", (T, Hv, Dv), xq.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, Hv, Dv, Dk), dtype=torch.float32, device=dev)
    if final_state is not None:
        _check(final_state, "final_state", (N, Hv, Dv, Dk), torch.float32, dev)
    ws_bytes = 0
    if workspace is not None:
        ws_bytes = workspace.numel() * workspace.element_size()
    else:
        need = int(lib.gdn_prefill_conv_workspace_bytes(N, T, Hqk, Hv, Dk, Dv))
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            ws_bytes = need
    rc = lib.gdn_prefill_conv(_ptr(xq), _ptr(xk), _ptr(xv), DTYPE[xq.dtype], _ptr(wq), _ptr(wk),
                              _ptr(wv), _ptr(conv_state), _ptr(conv_state_out), _ptr(g), _ptr(beta),
                              _ptr(initial_state), _ptr(cu_seqlens), N, T, Hqk, Hv, Dk, Dv, 0,
                              _ptr(o), _ptr(final_state), _ptr(workspace), ws_bytes,
                              _ptr(error_flag), _stream(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_prefill_conv")
    if conv_state_out is not None:
        return o, final_state, conv_state_out
    return o, final_state
