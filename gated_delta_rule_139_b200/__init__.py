"""Python binding of libkda.so -- the KDA chunked forward pass on B200 (sm_100a).

Thin ctypes marshalling around the C ABI of ``include/kda.h``; every step of the
computation runs in the library's CUDA kernels.  PyTorch provides device memory
and streams only.  If ``libkda.so`` has not been built this module raises on
first use: there is no fallback implementation.

    from gated_delta_rule_139_b200 import kda_fwd
    out, final_state = kda_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens)

Shapes (row-major): q, k [B,T,H,d_k]; v [B,T,H,d_v]; log_alpha [B,T,H,d_k] fp32;
beta [B,T,H] fp32; states [N,H,d_k,d_v] fp32; packed input passes [T,H,*]
tensors (or B=1) with cu_seqlens int32 [N+1].
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["kda_fwd", "kda_fwd_host", "kda_fwd_noalloc", "kda_fwd_snap", "kda_decode",
           "kda_transition", "kda_apply_transitions", "span_workspace", "kda_span_transition",
           "kda_span_forward", "kda_chunk_operands", "KDAError", "library_path", "load_library",
           "last_launch_count", "last_path", "check_device", "profile_enable", "profile_read",
           "STATUS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_LIBRARY selects another build of the same library (e.g. the phase-trace build)
library_path = os.environ.get("KDA_LIBRARY") or os.path.join(_PKG, "libkda.so")

STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
          3: "KDA_ERR_MISALIGNED", 4: "KDA_ERR_ALIAS", 5: "KDA_ERR_CUDA",
          6: "KDA_ERR_DEVICE_TIMEOUT"}
KDA_F32, KDA_BF16 = 0, 1


class KDAError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{self.name}: {detail}")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("qkv_dtype", ctypes.c_int32)]


class SnapSpec(ctypes.Structure):
    _fields_ = [("interval", ctypes.c_int32), ("max_snaps", ctypes.c_int32),
                ("num_slots", ctypes.c_int32)]


class FwdOpts(ctypes.Structure):
    _fields_ = [("out_gate", ctypes.c_void_p), ("snap", ctypes.POINTER(SnapSpec)),
                ("snap_slots", ctypes.c_void_p), ("snap_pool", ctypes.c_void_p)]


class DecodeDims(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("num_slots", ctypes.c_int32),
                ("qkv_dtype", ctypes.c_int32)]


_lib = None


def load_library():
    """Load libkda.so (raises if it is missing: build it with ``build.py``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError(f"{library_path} is missing; run "
                              "`python -m gated_delta_rule_139_b200.build` first")
        lib = ctypes.CDLL(library_path)
        p = ctypes.c_void_p
        sig = [p, p, p, p, p, p, p, ctypes.c_int32, p, p, ctypes.POINTER(Dims), p]
        for name in ("kda_fwd", "kda_fwd_host", "kda_fwd_noalloc"):
            fn = getattr(lib, name)
            fn.argtypes = sig
            fn.restype = ctypes.c_int
        lib.kda_fwd_snap.argtypes = sig[:-1] + [ctypes.POINTER(SnapSpec), p, p, p]
        lib.kda_fwd_snap.restype = ctypes.c_int
        lib.kda_fwd_ex.argtypes = sig[:-1] + [ctypes.POINTER(FwdOpts), p]
        lib.kda_fwd_ex.restype = ctypes.c_int
        lib.kda_decode.argtypes = [p, p, p, p, p, p, p, p, p, p, ctypes.POINTER(DecodeDims), p]
        lib.kda_transition.argtypes = [p, p, p, p, ctypes.POINTER(Dims), p, p]
        lib.kda_transition.restype = ctypes.c_int
        lib.kda_apply_transitions.argtypes = [p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              p, p, p]
        lib.kda_apply_transitions.restype = ctypes.c_int
        lib.kda_span_workspace_bytes.argtypes = [ctypes.POINTER(Dims)]
        lib.kda_span_workspace_bytes.restype = ctypes.c_size_t
        lib.kda_span_transition.argtypes = [p, p, p, p, p, ctypes.POINTER(Dims), p, ctypes.c_size_t, p,
                                            p]
        lib.kda_span_transition.restype = ctypes.c_int
        lib.kda_span_forward.argtypes = [p, p, p, p, p, p, p, p, ctypes.POINTER(Dims), p,
                                         ctypes.c_size_t, p]
        lib.kda_span_forward.restype = ctypes.c_int
        lib.kda_span_forward_ex.argtypes = lib.kda_span_forward.argtypes[:-1] + \
            [ctypes.POINTER(FwdOpts), p]
        lib.kda_span_forward_ex.restype = ctypes.c_int
        lib.kda_chunk_operands.argtypes = [p, p, p, p, p, ctypes.POINTER(Dims), p, p]
        lib.kda_chunk_operands.restype = ctypes.c_int
        lib.kda_selftest_wait.argtypes = [ctypes.c_uint64, ctypes.c_int32, p]
        lib.kda_selftest_wait.restype = ctypes.c_int
        lib.kda_decode.restype = ctypes.c_int
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_last_error.argtypes = []
        lib.kda_last_error.restype = ctypes.c_char_p
        lib.kda_last_launch_count.argtypes = []
        lib.kda_last_launch_count.restype = ctypes.c_int32
        lib.kda_last_path.argtypes = []
        lib.kda_last_path.restype = ctypes.c_char_p
        lib.kda_check_device.argtypes = [ctypes.c_void_p]
        lib.kda_check_device.restype = ctypes.c_int
        lib.kda_profile_enable.argtypes = [ctypes.c_int32]
        lib.kda_profile_enable.restype = None
        lib.kda_profile_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
        lib.kda_profile_read.restype = ctypes.c_int
        lib.kda_profile_slot_name.argtypes = [ctypes.c_int32]
        lib.kda_profile_slot_name.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def last_launch_count() -> int:
    """Kernel launches issued by the last kda_fwd call on this thread."""
    return int(load_library().kda_last_launch_count())


def last_path() -> str:
    """Kernel family of the last call on this thread ("ffma", "tc" or "decode")."""
    return load_library().kda_last_path().decode()


def profile_enable(on: bool = True) -> None:
    """Turn on/off CUDA-event timing of every internal kernel launch."""
    load_library().kda_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel name: (summed ms, launches)} since the previous read (synchronises)."""
    lib = load_library()
    n = 7
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib.kda_profile_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p), n))
    return {lib.kda_profile_slot_name(i).decode(): (ms[i], cnt[i]) for i in range(n) if cnt[i]}


def check_device(stream=None) -> None:
    """Synchronise ``stream`` and raise KDAError if a kernel recorded a device-side
    error (a bounded wait that gave up, or a malformed cu_seqlens table)."""
    s = None if stream is None else ctypes.c_void_p(stream.cuda_stream)
    _check(load_library().kda_check_device(s))


def _check(rc: int):
    if rc != 0:
        raise KDAError(rc, load_library().kda_last_error().decode())


def _dims(q_shape, v_shape, T_override, cu_len, bf16):
    if len(q_shape) == 4:
        B, T, H, dk = q_shape
    elif len(q_shape) == 3:
        B, (T, H, dk) = 1, q_shape
    else:
        raise ValueError("q must be [B,T,H,d_k] or [T,H,d_k]")
    return Dims(B, T, H, dk, v_shape[-1], max(cu_len - 1, 0) if cu_len else 0,
                KDA_BF16 if bf16 else KDA_F32)


def kda_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk: int = 64,
            out=None, final_state=None, stream=None, want_final: bool = True,
            out_gate=None, _entry: str = "kda_fwd", _snap=None):
    """KDA forward on CUDA tensors; returns (out, final_state or None).

    q/k/v are bf16 or fp32 CUDA tensors; gates and states fp32.  ``stream`` is a
    torch.cuda.Stream (default: the current stream).  Outputs are allocated when
    not given.  Runs asynchronously on the stream.  ``out_gate`` (same shape and
    dtype as out) multiplies the output before it is stored (kda_fwd_ex).
    """
    import torch

    lib = load_library()
    bf16 = q.dtype == torch.bfloat16
    if not bf16 and q.dtype != torch.float32:
        raise TypeError("q/k/v must be bfloat16 or float32")
    for t in (q, k, v, log_alpha, beta):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    d = _dims(tuple(q.shape), tuple(v.shape), None,
              cu_seqlens.numel() if cu_seqlens is not None else 0, bf16)
    N = d.num_seqs if cu_seqlens is not None else d.B
    if out is None:
        out = torch.empty(tuple(q.shape[:-1]) + (d.d_v,), dtype=q.dtype, device=q.device)
    if final_state is None and want_final:
        final_state = torch.empty((N, d.H, d.d_k, d.d_v), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    args = (ptr(q), ptr(k), ptr(v), ptr(log_alpha), ptr(beta), ptr(initial_state),
            ptr(cu_seqlens), int(chunk), ptr(out), ptr(final_state), ctypes.byref(d))
    if out_gate is not None or _snap is not None:
        if _entry != "kda_fwd":
            raise ValueError(f"{_entry} takes no output gate or snapshots")
        if out_gate is not None:
            if not out_gate.is_cuda or not out_gate.is_contiguous() or out_gate.dtype != q.dtype \
                    or tuple(out_gate.shape) != tuple(out.shape):
                raise ValueError("out_gate must be a contiguous CUDA tensor shaped and typed as out")
        opts = FwdOpts(None if out_gate is None else out_gate.data_ptr(), None, None, None)
        if _snap is not None:
            spec, slots, pool = _snap
            opts.snap = ctypes.pointer(spec)
            opts.snap_slots = slots.data_ptr()
            opts.snap_pool = pool.data_ptr()
        rc = lib.kda_fwd_ex(*args, ctypes.byref(opts), ctypes.c_void_p(stream.cuda_stream))
    else:
        rc = getattr(lib, _entry)(*args, ctypes.c_void_p(stream.cuda_stream))
    _check(rc)
    return out, final_state


def _snap_spec(snap_interval, snap_slots, snap_pool, n_seqs):
    import torch
    for t in (snap_slots, snap_pool):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("snap_slots and snap_pool must be contiguous CUDA tensors")
    if snap_slots.dtype != torch.int32 or snap_slots.dim() != 2:
        raise ValueError("snap_slots must be an int32 [N, max_snaps] tensor")
    if snap_slots.shape[0] != n_seqs:
        raise ValueError(f"snap_slots has {snap_slots.shape[0]} rows for {n_seqs} sequences")
    return SnapSpec(int(snap_interval), snap_slots.shape[1], snap_pool.shape[0])


def kda_fwd_snap(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, *,
                 snap_interval: int, snap_slots, snap_pool, chunk: int = 64, out=None,
                 final_state=None, stream=None, want_final: bool = True, out_gate=None):
    """kda_fwd that also writes prefix-cache state snapshots.

    Snapshot j of sequence n -- the state after its first (j+1)*snap_interval
    tokens (snap_interval a multiple of 64) -- goes to row snap_slots[n, j] of
    ``snap_pool`` [num_slots,H,d_k,d_v] fp32 when that entry is >= 0.
    ``snap_slots`` is an int32 CUDA tensor [N, max_snaps].  Returns (out,
    final_state or None); the pool is written in place.
    """
    n_seqs = (cu_seqlens.numel() - 1) if cu_seqlens is not None else q.shape[0]
    spec = _snap_spec(snap_interval, snap_slots, snap_pool, n_seqs)
    return kda_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out, final_state,
                   stream, want_final, out_gate=out_gate, _snap=(spec, snap_slots, snap_pool))


def kda_fwd_noalloc(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                    chunk: int = 64, out=None, final_state=None, stream=None,
                    want_final: bool = True):
    """kda_fwd through the entry point that allocates no device memory.

    The library's temporaries come from its fixed 32 MiB device scratch array
    instead of a memory pool (for callers that cannot allocate on the call
    path).  ``out`` and ``final_state`` are allocated here when not given (by
    torch, before the call); pass them in to keep the whole call free of
    allocations.  Calls that overlap on the GPU share the array and race.
    """
    return kda_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                   final_state, stream, want_final, _entry="kda_fwd_noalloc")


def kda_fwd_host(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                 chunk: int = 64, out=None, final_state=None, stream=None,
                 want_final: bool = True):
    """KDA forward on HOST numpy arrays (or CPU tensors; pinned memory copies
    asynchronously).  The library copies inputs in, runs, copies results back
    and synchronises; one long sequence (B = 1, no cu_seqlens) runs as a
    pipeline of spans so that the two copy directions overlap (kda_fwd_host).
    bf16 data is passed as uint16 bit patterns (numpy) or torch.bfloat16 CPU
    tensors.  Returns (out, final_state or None) on the host.
    """
    import numpy as np

    lib = load_library()

    def info(a):
        if a is None:
            return None, None, None
        if isinstance(a, np.ndarray):
            return a.ctypes.data, a.shape, a.dtype
        return a.data_ptr(), tuple(a.shape), a.dtype  # torch CPU tensor

    _, qs, qd = info(q)
    _, vs, _ = info(v)
    bf16 = str(qd) in ("uint16", "torch.bfloat16")
    cu_len = 0 if cu_seqlens is None else len(cu_seqlens)
    d = _dims(tuple(qs), tuple(vs), None, cu_len, bf16)
    N = d.num_seqs if cu_seqlens is not None else d.B
    if isinstance(q, np.ndarray):
        if out is None:
            out = np.empty(tuple(qs[:-1]) + (d.d_v,), dtype=q.dtype)
        if final_state is None and want_final:
            final_state = np.empty((N, d.H, d.d_k, d.d_v), dtype=np.float32)
        if cu_seqlens is not None:
            cu_seqlens = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    else:
        import torch
        if out is None:
            out = torch.empty(tuple(qs[:-1]) + (d.d_v,), dtype=q.dtype, pin_memory=q.is_pinned())
        if final_state is None and want_final:
            final_state = torch.empty((N, d.H, d.d_k, d.d_v), dtype=torch.float32,
                                      pin_memory=q.is_pinned())
    h = lambda a: None if a is None else ctypes.c_void_p(info(a)[0])
    s = None if stream is None else ctypes.c_void_p(stream.cuda_stream)
    rc = lib.kda_fwd_host(h(q), h(k), h(v), h(log_alpha), h(beta), h(initial_state),
                          h(cu_seqlens), int(chunk), h(out), h(final_state), ctypes.byref(d), s)
    _check(rc)
    return out, final_state


def kda_decode(q, k, v, log_alpha, beta, state, slots=None, out=None, token_states=None,
               want_token_states: bool = False, stream=None, out_gate=None):
    """Decode / multi-token verify step: T new tokens per sequence on a resident
    state, which is updated IN PLACE.  Returns (out, token_states or None).

    q, k [N,T,H,d_k]; v [N,T,H,d_v] (bf16 or fp32); log_alpha [N,T,H,d_k] and
    beta [N,T,H] fp32; state [S,H,d_k,d_v] fp32 where S = N, or the pool size
    when ``slots`` (int32 [N] on the device; -1 = padding entry) maps sequences
    to pool rows.  ``token_states`` [N,T,H,d_k,d_v] receives the state after
    every token (allocated here when ``want_token_states``).  ``out_gate``
    [N,T,H,d_v] (dtype of q) multiplies the output before it is stored.
    """
    import torch

    lib = load_library()
    bf16 = q.dtype == torch.bfloat16
    if not bf16 and q.dtype != torch.float32:
        raise TypeError("q/k/v must be bfloat16 or float32")
    for t in (q, k, v, log_alpha, beta, state):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if q.dim() != 4:
        raise ValueError("q must be [N,T,H,d_k]")
    N, T, H, dk = q.shape
    dv = v.shape[-1]
    d = DecodeDims(N, T, H, dk, dv, state.shape[0] if slots is not None else N,
                   KDA_BF16 if bf16 else KDA_F32)
    if out is None:
        out = torch.empty((N, T, H, dv), dtype=q.dtype, device=q.device)
    if token_states is None and want_token_states:
        token_states = torch.empty((N, T, H, dk, dv), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    if out_gate is not None and (not out_gate.is_cuda or not out_gate.is_contiguous()
                                 or out_gate.dtype != q.dtype
                                 or tuple(out_gate.shape) != tuple(out.shape)):
        raise ValueError("out_gate must be a contiguous CUDA tensor shaped and typed as out")
    rc = lib.kda_decode(ptr(q), ptr(k), ptr(v), ptr(log_alpha), ptr(beta), ptr(state), ptr(slots),
                        ptr(out), ptr(out_gate), ptr(token_states), ctypes.byref(d),
                        ctypes.c_void_p(stream.cuda_stream))
    _check(rc)
    return out, token_states


def kda_transition(k, v, log_alpha, beta, out=None, stream=None):
    """Affine map S_out = M S_in + B of each of the B sequences of [B,T,H,128]
    bf16 k, v (fp32 log_alpha, beta): returns trans [B,H,2,128,128] fp32 with
    trans[b,h,0] = B^T and trans[b,h,1] = M^T."""
    import torch

    lib = load_library()
    for t in (k, v, log_alpha, beta):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if k.dim() != 4:
        raise ValueError("k must be [B,T,H,128]")
    B, T, H, dk = k.shape
    d = Dims(B, T, H, dk, v.shape[-1], 0, KDA_BF16 if k.dtype == torch.bfloat16 else KDA_F32)
    if out is None:
        out = torch.empty((B, H, 2, 128, 128), dtype=torch.float32, device=k.device)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    _check(lib.kda_transition(ptr(k), ptr(v), ptr(log_alpha), ptr(beta), ctypes.byref(d),
                              ptr(out), ctypes.c_void_p(stream.cuda_stream)))
    return out


def kda_apply_transitions(trans, initial_state=None, out=None, stream=None):
    """State after a chain of spans: trans [count,B,H,2,128,128] (span 0 first),
    initial_state [B,H,128,128] or None (zero).  Returns [B,H,128,128] fp32."""
    import torch

    lib = load_library()
    if trans.dim() != 6 or not trans.is_cuda or not trans.is_contiguous():
        raise ValueError("trans must be a contiguous CUDA tensor [count,B,H,2,128,128]")
    count, B, H = trans.shape[:3]
    if out is None:
        out = torch.empty((B, H, 128, 128), dtype=torch.float32, device=trans.device)
    if stream is None:
        stream = torch.cuda.current_stream(trans.device)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    _check(lib.kda_apply_transitions(ptr(trans) if count else None, count, B, H,
                                     ptr(initial_state), ptr(out),
                                     ctypes.c_void_p(stream.cuda_stream)))
    return out


def _span_dims(k):
    import torch
    if k.dim() != 4:
        raise ValueError("k must be [B,T,H,128]")
    B, T, H, dk = k.shape
    return Dims(B, T, H, dk, dk, 0, KDA_BF16 if k.dtype == torch.bfloat16 else KDA_F32)


def span_workspace(k):
    """A device buffer for kda_span_transition / kda_span_forward on spans shaped like k."""
    import torch
    n = int(load_library().kda_span_workspace_bytes(ctypes.byref(_span_dims(k))))
    if n == 0:
        raise ValueError("invalid span dims")
    return torch.empty(n, dtype=torch.uint8, device=k.device)


def kda_span_transition(q, k, v, log_alpha, beta, workspace, out=None, stream=None):
    """kda_transition that also leaves the span's segment transitions and every
    chunk's output-pass operands (hence q) in ``workspace`` (from
    :func:`span_workspace`) for :func:`kda_span_forward`."""
    import torch
    lib = load_library()
    d = _span_dims(k)
    if out is None:
        out = torch.empty((d.B, d.H, 2, 128, 128), dtype=torch.float32, device=k.device)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    _check(lib.kda_span_transition(None if q is None else ptr(q), ptr(k), ptr(v), ptr(log_alpha),
                                   ptr(beta), ctypes.byref(d),
                                   ptr(workspace), workspace.numel(), ptr(out),
                                   ctypes.c_void_p(stream.cuda_stream)))
    return out


def kda_span_forward(q, k, v, log_alpha, beta, workspace, initial_state=None, out=None,
                     final_state=None, stream=None, want_final: bool = True, out_gate=None, *,
                     snap_interval=None, snap_slots=None, snap_pool=None):
    """kda_fwd on a span whose kda_span_transition filled ``workspace``.
    ``out_gate`` as in :func:`kda_fwd`; the snapshot arguments as in
    :func:`kda_fwd_snap`, with positions counted from the span's start
    (kda_span_forward_ex)."""
    import torch
    lib = load_library()
    d = _dims(tuple(q.shape), tuple(v.shape), None, 0, q.dtype == torch.bfloat16)
    if out is None:
        out = torch.empty(tuple(q.shape[:-1]) + (d.d_v,), dtype=q.dtype, device=q.device)
    if final_state is None and want_final:
        final_state = torch.empty((d.B, d.H, d.d_k, d.d_v), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    args = (ptr(q), ptr(k), ptr(v), ptr(log_alpha), ptr(beta), ptr(initial_state), ptr(out),
            ptr(final_state), ctypes.byref(d), ptr(workspace), workspace.numel())
    if out_gate is None and snap_interval is None:
        _check(lib.kda_span_forward(*args, ctypes.c_void_p(stream.cuda_stream)))
        return out, final_state
    opts = FwdOpts(None, None, None, None)
    if out_gate is not None:
        if not out_gate.is_cuda or not out_gate.is_contiguous() or out_gate.dtype != q.dtype \
                or tuple(out_gate.shape) != tuple(out.shape):
            raise ValueError("out_gate must be a contiguous CUDA tensor shaped and typed as out")
        opts.out_gate = out_gate.data_ptr()
    if snap_interval is not None:
        spec = _snap_spec(snap_interval, snap_slots, snap_pool, q.shape[0])
        opts.snap = ctypes.pointer(spec)
        opts.snap_slots = snap_slots.data_ptr()
        opts.snap_pool = snap_pool.data_ptr()
    _check(lib.kda_span_forward_ex(*args, ctypes.byref(opts), ctypes.c_void_p(stream.cuda_stream)))
    return out, final_state


CHUNK_IMAGE_BYTES = 74240


def kda_chunk_operands(q, k, v, log_alpha, beta, out=None, stream=None):
    """Every chunk's operand images as the forward pass computes them
    (kda_chunk_operands): a uint8 tensor [B * ceil(T/64) * H, 74240], entry
    (b * ceil(T/64) + c) * H + h for chunk c of sequence b and head h."""
    import torch
    lib = load_library()
    d = _span_dims(k)
    nch = (d.T + 63) // 64
    if out is None:
        out = torch.empty((d.B * nch * d.H, CHUNK_IMAGE_BYTES), dtype=torch.uint8, device=k.device)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    _check(lib.kda_chunk_operands(ptr(q), ptr(k), ptr(v), ptr(log_alpha), ptr(beta), ctypes.byref(d),
                                  ptr(out), ctypes.c_void_p(stream.cuda_stream)))
    return out
