"""fp64 CPU oracle for the KDA forward pass -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It is the independent checker of the
CUDA library: it shares no code with ``gated_delta_rule_139_b200`` and never
imports it.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, pthreads), built by
:func:`build` into ``libkda_oracle.so`` next to this file.  It follows the
delta-rule state update of aiblin.ru, "Kimi K3 -- открытая модель, которая
обошла закрытых лидеров рынка", section "Как хранить миллион токенов в памяти"
(partial erase then write of a fixed d_k x d_v state, write strength beta,
per-channel forget gate alpha clamped to [e^-5, 1]), read as

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t.

:func:`recurrent` evaluates that definition token by token; :func:`chunked`
evaluates the chunkwise reformulation of section "Как распараллелили
последовательное обновление" of the same page.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile kda_oracle.c with gcc into libkda_oracle.so (in place)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.kda_oracle_recurrent.argtypes = [p, p, p, i32, p, p, p, p, i64, i64, i64, i64, i64,
                                             p, i64, p, i32]
        lib.kda_oracle_recurrent.restype = i32
        lib.kda_oracle_chunked.argtypes = [p, p, p, i32, p, p, p, p, i64, i64, i64, i64, i64, i64,
                                           p, i64, p, i32]
        lib.kda_oracle_chunked.restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prep(q, k, v, log_alpha, beta, initial_state, cu_seqlens):
    """Flatten [B,T,H,d] / [T,H,d] inputs to the packed layout the C code reads.

    q, k, v are float32 arrays (exact values) or uint16 arrays holding bf16 bits.
    Returns (arrays..., cu int64, N, T, H, dk, dv, dtype_code, out_shape_prefix).
    """
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if q.dtype == np.float32:
        code = 0
    elif q.dtype == np.uint16:
        code = 1
    else:
        raise TypeError("q/k/v must be float32 or uint16 (bf16 bits)")
    if not (k.dtype == q.dtype and v.dtype == q.dtype):
        raise TypeError("q, k, v must share one dtype")
    lead = q.shape[:-2]
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    T = int(np.prod(lead))
    if cu_seqlens is None:
        if q.ndim == 4:
            B, Tb = q.shape[0], q.shape[1]
        else:
            B, Tb = 1, q.shape[0]
        cu = np.arange(B + 1, dtype=np.int64) * Tb
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    la = np.ascontiguousarray(log_alpha, dtype=np.float32)
    be = np.ascontiguousarray(beta, dtype=np.float32)
    s0 = None if initial_state is None else np.ascontiguousarray(initial_state, dtype=np.float32)
    if la.size != T * H * dk or be.size != T * H or v.size != T * H * dv or k.size != q.size:
        raise ValueError("inconsistent shapes")
    if s0 is not None and s0.size != N * H * dk * dv:
        raise ValueError("initial_state must be [N,H,dk,dv]")
    return q, k, v, la, be, s0, cu, N, T, H, dk, dv, code, lead


def _widen(a):
    """Exact fp64 copy of an fp32 array or of bf16 bit patterns (uint16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _run(fn_name, q, k, v, log_alpha, beta, initial_state, cu_seqlens, o_tokens, threads,
         chunk=None, out_gate=None):
    q, k, v, la, be, s0, cu, N, T, H, dk, dv, code, lead = _prep(
        q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    o_tokens = T if o_tokens is None else int(o_tokens)
    o = np.empty((max(o_tokens, 0), H, dv), dtype=np.float64)
    sf = np.empty((N, H, dk, dv), dtype=np.float64)
    lib = _load()
    args = [_ptr(q), _ptr(k), _ptr(v), code, _ptr(la), _ptr(be), _ptr(s0), _ptr(cu), N, T, H,
            dk, dv]
    if chunk is not None:
        args.append(int(chunk))
    args += [_ptr(o) if o_tokens > 0 else None, o_tokens, _ptr(sf), int(threads)]
    rc = getattr(lib, fn_name)(*args)
    if rc != 0:
        raise ValueError(f"{fn_name} rejected its arguments (code {rc})")
    if out_gate is not None and o_tokens > 0:
        # the output gate of a KDA block (aiblin.ru page, description of the layer
        # stack): a share of each output element passes on, o * gate, after the
        # attention and outside the recurrence
        g = _widen(out_gate)
        if g.size != T * H * dv:
            raise ValueError("out_gate must have the shape of the output")
        o *= g.reshape(T, H, dv)[:o_tokens]
    if o_tokens == T and len(lead) == 2:
        o = o.reshape(lead + (H, dv))
    return o, sf


def recurrent(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, o_tokens=None,
              threads=0, out_gate=None):
    """Token-by-token fp64 evaluation of the KDA recurrence.

    Returns (o, final_state): o is float64 [.., H, d_v] for the first ``o_tokens``
    packed tokens (all by default), final_state float64 [N, H, d_k, d_v].  With
    ``out_gate`` (shape of the output; fp32 or bf16 bits) o is multiplied by it.
    """
    return _run("kda_oracle_recurrent", q, k, v, log_alpha, beta, initial_state, cu_seqlens,
                o_tokens, threads, out_gate=out_gate)


def chunked(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk=64,
            o_tokens=None, threads=0, out_gate=None):
    """Chunkwise fp64 reformulation (plain exp(+-g), any chunk size >= 1)."""
    return _run("kda_oracle_chunked", q, k, v, log_alpha, beta, initial_state, cu_seqlens,
                o_tokens, threads, chunk=chunk, out_gate=out_gate)


def chunk_operands(q, k, v, log_alpha, beta, chunk=64):
    """Per-chunk operands of the chunkwise form, fp64, for ONE sequence.

    Same page and section as :func:`chunked` ("Как распараллелили последовательное
    обновление": all tokens of a chunk are processed together, then the state is handed
    on), with plain exp(+-g).  Inputs [T, H, *] or [1, T, H, *] (bf16 as uint16 bits).
    For chunk c (tokens c*chunk ..) of head h -- a ragged last chunk padded with tokens
    whose k, q, v, beta and log alpha are zero, which act as identity steps:

        g      in-chunk inclusive cumsum of clamp(log alpha, -5, 0)        [C, d_k]
        A      strict_lower(diag(beta) (K e^g)(K e^-g)^T)                  [C, C]
        T      (I + A)^-1, by forward substitution                         [C, C]
        W      T diag(beta) (K e^g)                                        [C, d_k]
        U      T diag(beta) V                                              [C, d_v]
        P      lower_incl((Q e^g)(K e^-g)^T)                               [C, C]
        Qt     Q e^g                                                       [C, d_k]
        Kdec   K e^(g_last - g)                                            [C, d_k]
        gamma  e^(g_last)                                                  [d_k]

    returned as a dict of arrays [n_chunks, H, ...].  From the incoming state S
    (d_k x d_v) the chunk's outputs are Qt S + P (U - W S) and its outgoing state
    diag(gamma) S + Kdec^T (U - W S).
    """
    q, k, v, la, be = (_widen(x) for x in (q, k, v, log_alpha, beta))
    if q.ndim == 4:
        if q.shape[0] != 1:
            raise ValueError("chunk_operands takes one sequence")
        q, k, v, la, be = q[0], k[0], v[0], la[0], be[0]
    T, H, dk = q.shape
    dv = v.shape[-1]
    C = int(chunk)
    n = (T + C - 1) // C
    pad = n * C - T

    def padded(a):
        return np.concatenate([a, np.zeros((pad,) + a.shape[1:])], axis=0) if pad else a

    q, k, v, la, be = (padded(x) for x in (q, k, v, la, be))
    out = {name: np.empty((n, H) + shape) for name, shape in
           (("g", (C, dk)), ("A", (C, C)), ("T", (C, C)), ("W", (C, dk)), ("U", (C, dv)),
            ("P", (C, C)), ("Qt", (C, dk)), ("Kdec", (C, dk)), ("gamma", (dk,)))}
    for c in range(n):
        sl = slice(c * C, (c + 1) * C)
        for h in range(H):
            g = np.cumsum(np.clip(la[sl, h], -5.0, 0.0), axis=0)
            K, Q, V, b = k[sl, h], q[sl, h], v[sl, h], be[sl, h]
            Ke, Kh, Qe = K * np.exp(g), K * np.exp(-g), Q * np.exp(g)
            A = np.tril(b[:, None] * (Ke @ Kh.T), -1)
            Tm = np.zeros((C, C))
            for i in range(C):  # row i of T from the rows before it: (I + A) T = I
                Tm[i] = -A[i, :i] @ Tm[:i]
                Tm[i, i] = 1.0
            out["g"][c, h] = g
            out["A"][c, h] = A
            out["T"][c, h] = Tm
            out["W"][c, h] = Tm @ (b[:, None] * Ke)
            out["U"][c, h] = Tm @ (b[:, None] * V)
            out["P"][c, h] = np.tril(Qe @ Kh.T)
            out["Qt"][c, h] = Qe
            out["Kdec"][c, h] = K * np.exp(g[-1] - g)
            out["gamma"][c, h] = np.exp(g[-1])
    return out
