"""Host-side checks of libkda.so: it loads, exports every declared symbol, and
rejects bad arguments before any launch (fake, never-dereferenced pointers)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_139_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(kda_\w+)\s*\(", src, flags=re.M)
    return names


def test_library_exports_every_declared_function():
    lib = kda.load_library()
    names = declared_functions()
    assert {"kda_fwd", "kda_fwd_host", "kda_status_string", "kda_last_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    lib = kda.load_library()
    for code, name in kda.STATUS.items():
        assert lib.kda_status_string(code).decode() == name


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced


def call(dims, q=FAKE, k=FAKE + (1 << 30), v=FAKE + (2 << 30), la=FAKE + (3 << 30),
         be=FAKE + (4 << 30), s0=None, cu=None, chunk=64, out=FAKE + (5 << 30), sf=None):
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    rc = lib.kda_fwd(P(q), P(k), P(v), P(la), P(be), P(s0), P(cu), chunk, P(out), P(sf),
                     ctypes.byref(dims), None)
    return kda.STATUS[rc], lib.kda_last_error().decode()


def D(B=1, T=128, H=2, dk=128, dv=128, N=0, dt=1):
    return kda.Dims(B, T, H, dk, dv, N, dt)


def test_rejects_unsupported_shapes_and_chunk():
    assert call(D(dk=96))[0] == "KDA_ERR_UNSUPPORTED"
    assert call(D(dv=32))[0] == "KDA_ERR_UNSUPPORTED"
    assert call(D(), chunk=32)[0] == "KDA_ERR_UNSUPPORTED"


def test_rejects_invalid_arguments():
    assert call(D(B=0))[0] == "KDA_ERR_INVALID_ARG"
    assert call(D(T=-1))[0] == "KDA_ERR_INVALID_ARG"
    assert call(D(dt=7))[0] == "KDA_ERR_INVALID_ARG"
    assert call(D(), q=None)[0] == "KDA_ERR_INVALID_ARG"
    assert call(D(B=2, N=3), cu=FAKE + (7 << 30))[0] == "KDA_ERR_INVALID_ARG"  # packed needs B=1
    assert call(D(N=0), cu=FAKE + (7 << 30))[0] == "KDA_ERR_INVALID_ARG"
    lib = kda.load_library()
    assert kda.STATUS[lib.kda_fwd(None, None, None, None, None, None, None, 64, None, None,
                                  None, None)] == "KDA_ERR_INVALID_ARG"


def test_rejects_misaligned_pointers():
    st, msg = call(D(), k=FAKE + 8)
    assert st == "KDA_ERR_MISALIGNED" and "k " in msg + " "


def test_rejects_aliasing():
    assert call(D(), out=FAKE + 64)[0] == "KDA_ERR_ALIAS"  # out inside q
    s0 = FAKE + (6 << 30)
    assert call(D(), s0=s0, sf=s0 + 16)[0] == "KDA_ERR_ALIAS"  # partial state overlap
    assert call(D(), sf=FAKE + (4 << 30))[0] == "KDA_ERR_ALIAS"  # final_state over beta


def test_state_in_place_passes_host_checks():
    # final_state == initial_state is allowed; the call then fails only at the
    # device-accessibility check (the fake pointers are not device memory)
    s0 = FAKE + (6 << 30)
    st, msg = call(D(), s0=s0, sf=s0)
    assert st == "KDA_ERR_INVALID_ARG" and "device-accessible" in msg


def test_zero_length_is_accepted_by_host_checks():
    st, msg = call(D(T=0), q=None, k=None, v=None, la=None, be=None, out=None)
    assert st in ("KDA_OK", "KDA_ERR_CUDA")  # no device needed for T=0 validation


# ---------------------------------------------------------------- kda_decode arguments
def call_decode(dims, q=FAKE, k=FAKE + (1 << 30), v=FAKE + (2 << 30), la=FAKE + (3 << 30),
                be=FAKE + (4 << 30), st=FAKE + (6 << 30), slots=None, out=FAKE + (5 << 30),
                ts=None, gate=None):
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    rc = lib.kda_decode(P(q), P(k), P(v), P(la), P(be), P(st), P(slots), P(out), P(gate), P(ts),
                        ctypes.byref(dims), None)
    return kda.STATUS[rc], lib.kda_last_error().decode()


def DD(N=4, T=2, H=2, dk=128, dv=128, S=0, dt=1):
    return kda.DecodeDims(N, T, H, dk, dv, S, dt)


def test_decode_rejects_bad_arguments():
    assert call_decode(DD(N=-1))[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(T=-1))[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(H=0))[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(dt=3))[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(dk=32))[0] == "KDA_ERR_UNSUPPORTED"
    assert call_decode(DD(), st=None)[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(), v=None)[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(S=0), slots=FAKE + (7 << 30))[0] == "KDA_ERR_INVALID_ARG"
    assert call_decode(DD(), out=FAKE + (5 << 30) + 4)[0] == "KDA_ERR_MISALIGNED"
    assert call_decode(DD(S=8), slots=FAKE + (7 << 30) + 2)[0] == "KDA_ERR_MISALIGNED"
    lib = kda.load_library()
    assert kda.STATUS[lib.kda_decode(None, None, None, None, None, None, None, None, None, None,
                                     None, None)] == "KDA_ERR_INVALID_ARG"


def test_decode_rejects_aliasing():
    # out inside v; state inside k; token_states overlapping the state
    assert call_decode(DD(), out=FAKE + (2 << 30) + 256)[0] == "KDA_ERR_ALIAS"
    assert call_decode(DD(), st=FAKE + (1 << 30) + 256)[0] == "KDA_ERR_ALIAS"
    st, msg = call_decode(DD(), ts=FAKE + (6 << 30) + 4096)
    assert st == "KDA_ERR_ALIAS" and "token_states" in msg
    assert call_decode(DD(), gate=FAKE + (5 << 30) + 32)[0] == "KDA_ERR_ALIAS"  # gate inside out
    assert call_decode(DD(), gate=FAKE + (7 << 30) + 8)[0] == "KDA_ERR_MISALIGNED"


def test_decode_empty_batch_is_a_no_op():
    # nothing to do: no pointer is looked at, no launch
    assert call_decode(DD(N=0), q=None, k=None, v=None, la=None, be=None, st=None,
                       out=None)[0] == "KDA_OK"
    assert kda.last_launch_count() == 0


# ---------------------------------------------------------------- kda_fwd_snap arguments
def call_snap(spec, slots=FAKE + (8 << 30), pool=FAKE + (9 << 30), dims=None, out=FAKE + (5 << 30)):
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    d = dims or D()
    rc = lib.kda_fwd_snap(P(FAKE), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)), P(FAKE + (3 << 30)),
                          P(FAKE + (4 << 30)), None, None, 64, P(out), None, ctypes.byref(d),
                          None if spec is None else ctypes.byref(spec), P(slots), P(pool), None)
    return kda.STATUS[rc], lib.kda_last_error().decode()


def test_snap_rejects_bad_arguments():
    S = kda.SnapSpec
    assert call_snap(None)[0] == "KDA_ERR_INVALID_ARG"
    assert call_snap(S(0, 2, 4))[0] == "KDA_ERR_INVALID_ARG"
    assert call_snap(S(96, 2, 4))[0] == "KDA_ERR_INVALID_ARG"  # not a multiple of the chunk
    assert call_snap(S(64, -1, 4))[0] == "KDA_ERR_INVALID_ARG"
    assert call_snap(S(64, 2, 4), slots=None)[0] == "KDA_ERR_INVALID_ARG"
    assert call_snap(S(64, 2, 4), pool=FAKE + (9 << 30) + 4)[0] == "KDA_ERR_MISALIGNED"
    assert call_snap(S(64, 2, 4), slots=FAKE + (8 << 30) + 2)[0] == "KDA_ERR_MISALIGNED"
    # the forward's own checks still come first
    assert call_snap(S(64, 2, 4), dims=D(dk=96))[0] == "KDA_ERR_UNSUPPORTED"


def test_snap_rejects_aliasing():
    S = kda.SnapSpec
    st, msg = call_snap(S(64, 2, 4), pool=FAKE + (5 << 30))  # pool == out
    assert st == "KDA_ERR_ALIAS" and "snap_pool" in msg
    st, msg = call_snap(S(64, 2, 4), slots=FAKE + (5 << 30) + 64)  # slot table inside out
    assert st == "KDA_ERR_ALIAS"


# ---------------------------------------------------------------- kda_fwd_ex (output gate)
def call_ex(gate, out=FAKE + (5 << 30), dims=None):
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    opts = kda.FwdOpts(gate, None, None, None)
    d = dims or D()
    rc = lib.kda_fwd_ex(P(FAKE), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)), P(FAKE + (3 << 30)),
                        P(FAKE + (4 << 30)), None, None, 64, P(out), None, ctypes.byref(d),
                        ctypes.byref(opts), None)
    return kda.STATUS[rc], lib.kda_last_error().decode()


def test_gate_rejects_bad_pointers():
    assert call_ex(FAKE + (7 << 30) + 2)[0] == "KDA_ERR_MISALIGNED"
    st, msg = call_ex(FAKE + (5 << 30) + 64)  # gate inside out
    assert st == "KDA_ERR_ALIAS" and "out_gate" in msg
    assert call_ex(FAKE + (7 << 30), dims=D(dv=48))[0] == "KDA_ERR_UNSUPPORTED"


# ---------------------------------------------------------------- transitions (context parallel)
def test_transition_rejects_bad_arguments():
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(d, k=FAKE, v=FAKE + (1 << 30), la=FAKE + (2 << 30), be=FAKE + (3 << 30),
             tr=FAKE + (4 << 30)):
        rc = lib.kda_transition(P(k), P(v), P(la), P(be), ctypes.byref(d), P(tr), None)
        return kda.STATUS[rc]

    assert call(D(dk=64, dv=64)) == "KDA_ERR_UNSUPPORTED"
    assert call(D(dt=0)) == "KDA_ERR_UNSUPPORTED"  # fp32 inputs
    assert call(D(B=0)) == "KDA_ERR_INVALID_ARG"
    assert call(D(), tr=None) == "KDA_ERR_INVALID_ARG"
    assert call(D(), v=None) == "KDA_ERR_INVALID_ARG"
    assert call(D(), tr=FAKE + (4 << 30) + 8) == "KDA_ERR_MISALIGNED"
    assert call(D(), tr=FAKE + (1 << 30) + 1024) == "KDA_ERR_ALIAS"  # trans inside v


def test_apply_transitions_rejects_bad_arguments():
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(count=2, B=1, H=2, tr=FAKE, s0=FAKE + (1 << 30), out=FAKE + (2 << 30)):
        return kda.STATUS[lib.kda_apply_transitions(P(tr), count, B, H, P(s0), P(out), None)]

    assert call(count=-1) == "KDA_ERR_INVALID_ARG"
    assert call(H=0) == "KDA_ERR_INVALID_ARG"
    assert call(tr=None) == "KDA_ERR_INVALID_ARG"
    assert call(out=None) == "KDA_ERR_INVALID_ARG"
    assert call(out=FAKE + (2 << 30) + 4) == "KDA_ERR_MISALIGNED"
    assert call(out=FAKE + 4096) == "KDA_ERR_ALIAS"  # state_out inside trans
    assert call(out=FAKE + (1 << 30) + 4096) == "KDA_ERR_ALIAS"  # partial overlap with s0


# ---------------------------------------------------------------- span workspace (context parallel)
def test_span_workspace_size_and_bad_arguments():
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    n = lib.kda_span_workspace_bytes(ctypes.byref(D(B=1, T=1 << 16, H=8)))
    assert n > 0 and n % 256 == 0
    assert lib.kda_span_workspace_bytes(ctypes.byref(D(B=0))) == 0
    assert lib.kda_span_workspace_bytes(None) == 0

    def trans_call(ws=FAKE + (8 << 30), nbytes=n, d=None, q=FAKE + (9 << 30)):
        rc = lib.kda_span_transition(P(q), P(FAKE), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)),
                                     P(FAKE + (3 << 30)), ctypes.byref(d or D(T=1 << 16, H=8)),
                                     P(ws), nbytes, P(FAKE + (4 << 30)), None)
        return kda.STATUS[rc]

    assert trans_call(q=None) == "KDA_ERR_INVALID_ARG"  # the workspace needs q
    assert trans_call(q=FAKE + (9 << 30) + 8) == "KDA_ERR_MISALIGNED"
    assert trans_call(ws=FAKE + (9 << 30)) == "KDA_ERR_ALIAS"  # workspace over q

    assert trans_call(ws=None) == "KDA_ERR_INVALID_ARG"
    assert trans_call(ws=FAKE + (8 << 30) + 16) == "KDA_ERR_MISALIGNED"
    assert trans_call(nbytes=n - 256) == "KDA_ERR_INVALID_ARG"
    assert trans_call(ws=FAKE + (1 << 30)) == "KDA_ERR_ALIAS"  # workspace over v
    assert trans_call(d=D(T=1 << 16, H=8, dk=64, dv=64)) == "KDA_ERR_UNSUPPORTED"

    def fwd_call(ws=FAKE + (8 << 30), nbytes=n, d=None):
        rc = lib.kda_span_forward(P(FAKE), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)),
                                  P(FAKE + (3 << 30)), P(FAKE + (4 << 30)), None,
                                  P(FAKE + (5 << 30)), None, ctypes.byref(d or D(T=1 << 16, H=8)),
                                  P(ws), nbytes, None)
        return kda.STATUS[rc]

    assert fwd_call(d=D(T=1 << 16, H=8, dt=0)) in ("KDA_ERR_UNSUPPORTED", "KDA_ERR_INVALID_ARG")

    assert fwd_call(ws=FAKE + (8 << 30) + 16) == "KDA_ERR_MISALIGNED"
    assert fwd_call(nbytes=n - 256) == "KDA_ERR_INVALID_ARG"
    assert fwd_call(ws=FAKE + (5 << 30)) == "KDA_ERR_ALIAS"  # workspace over out


def test_span_forward_ex_checks_its_options():
    lib = kda.load_library()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    d = D(T=1 << 16, H=8)
    n = lib.kda_span_workspace_bytes(ctypes.byref(d))

    def call_ex(opts, ws=FAKE + (8 << 30)):
        rc = lib.kda_span_forward_ex(P(FAKE), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)),
                                     P(FAKE + (3 << 30)), P(FAKE + (4 << 30)), None,
                                     P(FAKE + (5 << 30)), None, ctypes.byref(d), P(ws), n,
                                     None if opts is None else ctypes.byref(opts), None)
        return kda.STATUS[rc]

    gate = FAKE + (6 << 30)
    assert call_ex(kda.FwdOpts(gate + 8, None, None, None)) == "KDA_ERR_MISALIGNED"
    assert call_ex(kda.FwdOpts(FAKE + (5 << 30), None, None, None)) == "KDA_ERR_ALIAS"  # gate = out
    spec = kda.SnapSpec(100, 4, 8)  # interval not a multiple of 64
    assert call_ex(kda.FwdOpts(None, ctypes.pointer(spec), FAKE + (7 << 30),
                               FAKE + (9 << 30))) == "KDA_ERR_INVALID_ARG"
    spec = kda.SnapSpec(128, 4, 8)
    assert call_ex(kda.FwdOpts(None, ctypes.pointer(spec), FAKE + (7 << 30), None)) \
        == "KDA_ERR_INVALID_ARG"  # pool missing
    # workspace placed over the snapshot pool
    assert call_ex(kda.FwdOpts(None, ctypes.pointer(spec), FAKE + (7 << 30), FAKE + (8 << 30)),
                   ws=FAKE + (8 << 30)) == "KDA_ERR_ALIAS"


# ---------------------------------------------------------------- host and no-allocation entry points
@pytest.mark.parametrize("entry", ["kda_fwd_host", "kda_fwd_noalloc"])
def test_host_and_noalloc_entry_points_reject_bad_arguments(entry):
    """The argument checks of kda_fwd hold for these entry points too, before any CUDA
    call (the pointers are never dereferenced)."""
    lib = kda.load_library()
    fn = getattr(lib, entry)
    P = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(d=None, q=FAKE, out=FAKE + (5 << 30), chunk=64, sf=None):
        rc = fn(P(q), P(FAKE + (1 << 30)), P(FAKE + (2 << 30)), P(FAKE + (3 << 30)), P(FAKE + (4 << 30)),
                None, None, chunk, P(out), P(sf), ctypes.byref(d or D()), None)
        return kda.STATUS[rc]

    assert call(d=D(dk=96)) == "KDA_ERR_UNSUPPORTED"
    assert call(chunk=32) == "KDA_ERR_UNSUPPORTED"
    assert call(d=D(B=0)) == "KDA_ERR_INVALID_ARG"
    assert call(q=None) == "KDA_ERR_INVALID_ARG"
    assert call(q=FAKE + 8) == "KDA_ERR_MISALIGNED"
    assert call(out=FAKE + (1 << 30)) == "KDA_ERR_ALIAS"  # out over k
    assert call(sf=FAKE + (4 << 30)) == "KDA_ERR_ALIAS"   # final_state over beta
