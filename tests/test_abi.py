"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments synchronously without touching a
GPU (every call below returns before any CUDA runtime call)."""
import ctypes
import os
import re

import pytest

import gated_deltanet_04_b200 as gdn
from gated_deltanet_04_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    gdn_build.build()
    return gdn.library()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", txt)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_prefill_ex", "gdn_decode_step", "gdn_prefill_workspace_bytes",
            "gdn_status_string", "gdn_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libgdn.so does not export {n}"


def test_status_strings_and_version(lib):
    for code, name in gdn.STATUS.items():
        assert lib.gdn_status_string(code).decode() == name
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version() >= 10000


def test_workspace_bytes_is_pure(lib):
    a = lib.gdn_prefill_workspace_bytes(1, 262144, 16, 48, 128, 128, 64)
    b = lib.gdn_prefill_workspace_bytes(1, 262144, 16, 48, 128, 128, 64)
    assert a == b and a >= 0


def test_conv_workspace_holds_pool_scratch_and_filters(lib):
    """gdn_prefill_conv's scratch: the pool kernel's, then one 2 KB filter block
    per q, k and v head; none for an empty call or an unsupported shape."""
    pool = lib.gdn_prefill_ex_workspace_bytes(1, 262144, 16, 48, 128, 128, 64, 4)
    conv = lib.gdn_prefill_conv_workspace_bytes(1, 262144, 16, 48, 128, 128)
    assert pool > 0 and conv >= pool + (2 * 16 + 48) * 2048
    assert conv - (2 * 16 + 48) * 2048 < pool + 256
    assert lib.gdn_prefill_conv_workspace_bytes(1, 0, 16, 48, 128, 128) == 0
    assert lib.gdn_prefill_conv_workspace_bytes(1, 4096, 16, 48, 64, 128) == 0
    assert lib.gdn_prefill_conv_workspace_bytes(2, 4096, 16, 48, 128, 128) == 0  # 96 units


def test_host_scratch_bytes(lib):
    """gdn_prefill_host's scratch: state, workspace and two segment buffers,
    growing with the segment length up to the sequence length; 0 for bad sizes."""
    per_token = 2 * (2 * 16 * 128 * 2 + 2 * 48 * 128 * 2 + 2 * 48 * 4)  # two buffers, bf16
    a = lib.gdn_prefill_host_scratch_bytes(262144, 16, 48, 128, 128, 64, 0, 16384)
    b = lib.gdn_prefill_host_scratch_bytes(262144, 16, 48, 128, 128, 64, 0, 32768)
    assert a >= 16384 * per_token + 48 * 128 * 128 * 4
    assert b - a >= 16384 * per_token
    assert lib.gdn_prefill_host_scratch_bytes(1000, 16, 48, 128, 128, 64, 0, 16384) == \
        lib.gdn_prefill_host_scratch_bytes(1000, 16, 48, 128, 128, 64, 0, 0)
    assert lib.gdn_prefill_host_scratch_bytes(-1, 16, 48, 128, 128, 64, 0, 0) == 0
    assert lib.gdn_prefill_host_scratch_bytes(100, 16, 48, 128, 128, 64, 5, 0) == 0


def test_host_prefill_rejects_bad_segments_before_any_copy(lib):
    """A segment length that is not a multiple of 64, or no scratch, fails
    validation without touching the (fake) pointers."""
    rc = lib.gdn_prefill_host(P, P, P, 0, P, P, None, 100, 16, 48, 128, 128, 64, P, None, 100, P,
                              1 << 40, None, None)
    assert rc == INVALID
    rc = lib.gdn_prefill_host(P, P, P, 0, P, P, None, 100, 16, 48, 128, 128, 64, P, None, 0, None,
                              0, None, None)
    assert rc == INVALID


# fake, 16-byte aligned "device" addresses: validation rejects the call before
# any of them could be dereferenced
P = 0x10000
MIS = 0x10008


def prefill(lib, **kw):
    args = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000, s0=None,
                cu=None, N=1, T=64, Hqk=16, Hv=48, Dk=128, Dv=128, chunk=64, o=P + 0x5000,
                sT=None, ws=None, wsb=0, err=None, stream=None)
    args.update(kw)
    return lib.gdn_prefill(args["q"], args["k"], args["v"], args["dt"], args["g"], args["beta"],
                           args["s0"], args["cu"], args["N"], args["T"], args["Hqk"], args["Hv"],
                           args["Dk"], args["Dv"], args["chunk"], args["o"], args["sT"], args["ws"],
                           args["wsb"], args["err"], args["stream"])


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID),
    (dict(o=None), INVALID),
    (dict(g=None), INVALID),
    (dict(q=MIS), INVALID),
    (dict(s0=MIS), INVALID),
    (dict(err=MIS), INVALID),
    (dict(dt=7), INVALID),
    (dict(N=-1), INVALID),
    (dict(T=-5), INVALID),
    (dict(Hv=47), INVALID),          # Hv % Hqk != 0
    (dict(Hqk=0), INVALID),
    (dict(N=2, cu=None), INVALID),   # several sequences need cu_seqlens
    (dict(o=P), INVALID),            # o aliases q
    (dict(chunk=-1), INVALID),
    (dict(Dk=96), UNSUPPORTED),
    (dict(Dv=256), UNSUPPORTED),
    (dict(chunk=128), UNSUPPORTED),
])
def test_prefill_rejects(lib, kw, code):
    assert prefill(lib, **kw) == code


def prefill_ex(lib, kernel, **kw):
    args = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000, s0=None,
                cu=None, N=1, T=64, Hqk=16, Hv=48, Dk=128, Dv=128, chunk=64, o=P + 0x5000,
                sT=None, ws=None, wsb=0, err=None, stream=None)
    args.update(kw)
    return lib.gdn_prefill_ex(args["q"], args["k"], args["v"], args["dt"], args["g"], args["beta"],
                              args["s0"], args["cu"], args["N"], args["T"], args["Hqk"], args["Hv"],
                              args["Dk"], args["Dv"], args["chunk"], args["o"], args["sT"],
                              args["ws"], args["wsb"], args["err"], args["stream"], kernel)


@pytest.mark.parametrize("kernel,kw,code", [
    (7, {}, INVALID),                              # no such kernel
    (4, dict(N=2, cu=P + 0x6000), UNSUPPORTED),    # the pool kernel takes at most 64 units
    (4, dict(dt=1), UNSUPPORTED),
    (1, dict(Dk=64, Dv=64), UNSUPPORTED),          # tensor-core kernels need D = 128
    (2, dict(dt=1), UNSUPPORTED),                  # ... and bf16
    (1, dict(chunk=32), UNSUPPORTED),              # ... and chunk 64
    (3, dict(q=None), INVALID),
])
def test_prefill_ex_rejects(lib, kernel, kw, code):
    lib.gdn_prefill_ex.argtypes = lib.gdn_prefill.argtypes + [ctypes.c_int]
    assert prefill_ex(lib, kernel, **kw) == code


def test_prefill_nothing_to_do_is_ok(lib):
    assert prefill(lib, N=0, T=0, cu=P + 0x6000) == 0
    assert prefill(lib, T=0, sT=None) == 0


def decode(lib, **kw):
    args = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000,
                state=P + 0x7000, N=256, Hqk=16, Hv=48, Dk=128, Dv=128, o=P + 0x5000, err=None,
                stream=None)
    args.update(kw)
    return lib.gdn_decode_step(args["q"], args["k"], args["v"], args["dt"], args["g"],
                               args["beta"], args["state"], args["N"], args["Hqk"], args["Hv"],
                               args["Dk"], args["Dv"], args["o"], args["err"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(state=None), INVALID),
    (dict(k=MIS), INVALID),
    (dict(o=P + 0x7000), INVALID),   # o aliases the state
    (dict(Hv=40), INVALID),
    (dict(dt=2), INVALID),
    (dict(Dk=24), UNSUPPORTED),
])
def test_decode_rejects(lib, kw, code):
    assert decode(lib, **kw) == code


def test_decode_empty_batch_is_ok(lib):
    assert decode(lib, N=0) == 0


def decode_bf16_state(lib, **kw):
    args = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000,
                state=P + 0x7000, N=256, Hqk=16, Hv=48, Dk=128, Dv=128, o=P + 0x5000, err=None,
                stream=None)
    args.update(kw)
    return lib.gdn_decode_step_bf16_state(args["q"], args["k"], args["v"], args["dt"], args["g"],
                                          args["beta"], args["state"], args["N"], args["Hqk"],
                                          args["Hv"], args["Dk"], args["Dv"], args["o"],
                                          args["err"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(state=None), INVALID),
    (dict(state=MIS), INVALID),
    (dict(o=P + 0x7000), INVALID),   # o aliases the state
    (dict(Hv=40), INVALID),
    (dict(dt=2), INVALID),
    (dict(Dk=64, Dv=64), UNSUPPORTED),   # the bfloat16 state kernel is D = 128 only
    (dict(Dv=96), UNSUPPORTED),
])
def test_decode_bf16_state_rejects(lib, kw, code):
    assert decode_bf16_state(lib, **kw) == code


def test_decode_bf16_state_empty_batch_is_ok(lib):
    assert decode_bf16_state(lib, N=0) == 0


def test_order_entry_points_reject_unknown_orders(lib):
    """gdn_prefill_order / gdn_decode_step_order: a gdn_order outside the enum is
    an argument error; the rest of the checks are those of the plain calls."""
    pf = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000, s0=None,
              cu=None, N=1, T=64, Hqk=16, Hv=48, Dk=128, Dv=128, chunk=64, o=P + 0x5000,
              sT=None, ws=None, wsb=0, err=None, stream=None)
    def prefill_order(order, **kw):
        a = dict(pf, **kw)
        return lib.gdn_prefill_order(a["q"], a["k"], a["v"], a["dt"], a["g"], a["beta"], a["s0"],
                                     a["cu"], a["N"], a["T"], a["Hqk"], a["Hv"], a["Dk"], a["Dv"],
                                     a["chunk"], a["o"], a["sT"], a["ws"], a["wsb"], a["err"],
                                     a["stream"], 3, order)  # kernel 3: recurrent (no workspace)
    assert prefill_order(2) == INVALID
    assert prefill_order(-1) == INVALID
    assert prefill_order(1, Hv=40) == INVALID
    assert prefill_order(1, Dk=24) == UNSUPPORTED
    assert prefill_order(1, N=0, T=0, cu=P + 0x6000) == 0

    def decode_order(order, **kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000,
                 state=P + 0x7000, N=256, Hqk=16, Hv=48, Dk=128, Dv=128, o=P + 0x5000)
        a.update(kw)
        return lib.gdn_decode_step_order(a["q"], a["k"], a["v"], a["dt"], a["g"], a["beta"],
                                         a["state"], a["N"], a["Hqk"], a["Hv"], a["Dk"], a["Dv"],
                                         a["o"], None, None, order)
    assert decode_order(2) == INVALID
    assert decode_order(1, k=MIS) == INVALID
    assert decode_order(1, Dk=24) == UNSUPPORTED
    assert decode_order(1, N=0) == 0


def decode_slots(lib, **kw):
    a = dict(q=P, k=P + 0x1000, v=P + 0x2000, dt=0, g=P + 0x3000, beta=P + 0x4000,
             pool=P + 0x7000, S=300, slot=P + 0x8000, reset=None, N=256, Hqk=16, Hv=48, Dk=128,
             Dv=128, o=P + 0x5000, err=None, stream=None)
    a.update(kw)
    return lib.gdn_decode_step_slots(a["q"], a["k"], a["v"], a["dt"], a["g"], a["beta"], a["pool"],
                                     a["S"], a["slot"], a["reset"], a["N"], a["Hqk"], a["Hv"],
                                     a["Dk"], a["Dv"], a["o"], a["err"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(slot=None), INVALID),
    (dict(pool=None), INVALID),
    (dict(S=0), INVALID),
    (dict(reset=MIS), INVALID),
    (dict(slot=MIS), INVALID),
    (dict(o=P + 0x7000), INVALID),   # o aliases the pool
    (dict(Hv=40), INVALID),
    (dict(Dk=24), UNSUPPORTED),
])
def test_decode_slots_rejects(lib, kw, code):
    assert decode_slots(lib, **kw) == code


def test_decode_slots_empty_batch_is_ok(lib):
    assert decode_slots(lib, N=0, S=0, slot=None) == 0


def short_conv(lib, **kw):
    a = dict(xq=P, xk=P + 0x1000, xv=P + 0x2000, dt=0, wq=P + 0x3000, wk=P + 0x4000,
             wv=P + 0x5000, sin=None, sout=None, cu=None, N=1, T=64, Hqk=16, Hv=48, Dk=128,
             Dv=128, q=P + 0x6000, k=P + 0x7000, v=P + 0x8000, err=None, stream=None)
    a.update(kw)
    return lib.gdn_short_conv_norm(a["xq"], a["xk"], a["xv"], a["dt"], a["wq"], a["wk"], a["wv"],
                                   a["sin"], a["sout"], a["cu"], a["N"], a["T"], a["Hqk"], a["Hv"],
                                   a["Dk"], a["Dv"], a["q"], a["k"], a["v"], a["err"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(xq=None), INVALID),
    (dict(wv=None), INVALID),
    (dict(xk=MIS), INVALID),
    (dict(sin=MIS), INVALID),
    (dict(q=P), INVALID),              # q aliases xq
    (dict(v=P + 0x6000), INVALID),     # v aliases q
    (dict(N=2), INVALID),              # no cu_seqlens with N != 1
    (dict(dt=2), INVALID),
    (dict(Dk=64, Dv=64), UNSUPPORTED),
])
def test_short_conv_norm_rejects(lib, kw, code):
    assert short_conv(lib, **kw) == code


def test_short_conv_norm_nothing_to_do_is_ok(lib):
    assert short_conv(lib, N=0, T=0, cu=P + 0x9000) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 2, 16)
    with pytest.raises(ValueError):
        gdn.gdn_prefill(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2))
    with pytest.raises(ValueError):
        gdn.gdn_decode_step(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2), torch.zeros(4, 2, 16, 16))


def test_product_path_never_imports_the_oracle():
    """The library binding and the CUDA sources must not reach the oracle."""
    pkg = os.path.join(ROOT, "gated_deltanet_04_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "gdn_oracle" not in txt, f


def test_header_compiles_as_c99_and_links(tmp_path):
    """A plain C caller: include/gdn.h compiles as C99 with warnings as errors,
    the program links against libgdn.so, and the host-only calls work (no GPU:
    an argument error returns before any CUDA call)."""
    import subprocess
    gdn_build.build()
    src = tmp_path / "caller.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "gdn.h"
int main(void) {
    if (gdn_version() < 10000) return 1;
    if (strcmp(gdn_status_string(GDN_ERR_BAD_SLOT), "GDN_ERR_BAD_SLOT") != 0) return 2;
    /* invalid enum: rejected synchronously */
    if (gdn_decode_step_order(0, 0, 0, GDN_DTYPE_BF16, 0, 0, 0, 1, 1, 1, 128, 128, 0, 0, 0,
                              (gdn_order)7) != GDN_ERR_INVALID_ARGUMENT) return 3;
    if (gdn_prefill_workspace_bytes(1, 4096, 16, 48, 128, 128, 64) == 0) return 4;
    printf("ok\n");
    return 0;
}
""")
    lib_dir = os.path.join(ROOT, "gated_deltanet_04_b200")
    exe = tmp_path / "caller"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", lib_dir, "-lgdn", "-Wl,-rpath," + lib_dir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_stall_entry_point_rejects_bad_settings(lib):
    """The timeout-test entry point refuses a negative unit or a non-positive
    limit before any CUDA call."""
    f = lib.gdn_debug_prefill_pool_stall
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                  vp, vp, vp, ctypes.c_size_t, vp, vp, i32, i64]
    f.restype = ctypes.c_int
    P = 0x10000
    args = [P, P + 0x1000, P + 0x2000, 0, P + 0x3000, P + 0x4000, None, None, 1, 64, 1, 3, 128,
            128, 64, P + 0x5000, None, P + 0x6000, 1 << 20, None, None]
    assert f(*args, -1, 1 << 20) == 1  # GDN_ERR_INVALID_ARGUMENT
    assert f(*args, 0, 0) == 1
