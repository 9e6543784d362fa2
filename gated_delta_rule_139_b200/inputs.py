"""Seeded synthetic inputs for the KDA forward pass.

This module only draws random numbers and shapes them; it holds none of the
recurrence's arithmetic.  It serves both the CUDA library's tests/benchmark and
the fp64 oracle, which receive the same arrays.

Recipes (the five forward workloads the library is measured and checked on):

  ``tiny_fp32``   B=1, H=1, T=256, d_k=d_v=64, fp32 q/k/v; q,k ~ N(0,1) then
                  L2-normalised per (token, head); v ~ N(0,1);
                  beta = sigmoid(N(0,1)); log_alpha = -softplus(N(0,1)) clamped
                  to [-5, 0]; zero initial state.
  ``b2_t4k``      B=2, H=8, T=4096, d=128, bf16 q/k/v, fp32 gates;
                  log_alpha = -softplus(N(0,2)) clamped; initial state ~ N(0,0.02).
  ``prefill_64k`` B=1, H=32, T=65536, d=128, bf16; distributions of ``tiny_fp32``
                  (zero initial state), plus 10% of the (head, channel) pairs
                  pinned to log_alpha = -5 and another 10% pinned to 0.
  ``packed_16``   16 sequences, lengths uniform on [1024, 32768], concatenated
                  (cu_seqlens), H=16, d=128, bf16; distributions of ``b2_t4k``;
                  one random initial state ~ N(0,0.02) per sequence.
  ``prefill_1m``  B=1, H=8, T=2^20, d=128, bf16; log_alpha = -softplus(N(-1,1))
                  clamped; zero initial state.

Two more recipes time the decode / multi-token verify step on resident states:

  ``decode_1024x1``  1024 sequences x 1 new token, H=8, d=128, bf16; gates of
                     ``prefill_1m``; states ~ N(0,0.3) (a state after a long
                     prefill holds O(1) entries).
  ``verify_512x4``   512 sequences x 4 drafted tokens, otherwise the same.

N(mu, sigma) means mean and standard deviation.  Every workload uses seed 0;
each tensor draws from its own child of ``np.random.SeedSequence(seed)`` in the
fixed order q, k, v, beta, log_alpha, initial state, lengths, pins.  Large
tensors are drawn in fixed blocks with per-block grandchild seeds, so the values
do not depend on the number of threads.

bf16 tensors are returned as uint16 bit patterns (round-to-nearest-even from the
fp32 draw); :func:`bf16_to_f32` widens them exactly.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

BLOCK = 1 << 22  # elements per independently seeded block


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _blocked(ss: np.random.SeedSequence, n: int, row: int, fn, out: np.ndarray):
    """Fill ``out.reshape(-1)`` block by block; ``fn(rng, count) -> values``.

    Blocks are multiples of ``row`` so per-row post-processing stays inside one
    block.
    """
    flat = out.reshape(-1)
    blk = max(row, (BLOCK // row) * row)
    nb = (n + blk - 1) // blk
    kids = ss.spawn(nb)

    def work(b):
        lo, hi = b * blk, min(n, (b + 1) * blk)
        flat[lo:hi] = fn(np.random.default_rng(kids[b]), hi - lo)

    if nb == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nb)))


def _unit_rows(d: int, bf16: bool):
    def fn(rng, count):
        x = rng.standard_normal(count, dtype=np.float32).reshape(-1, d)
        x /= np.sqrt(np.einsum("ij,ij->i", x, x, dtype=np.float32))[:, None]
        x = x.reshape(-1)
        return f32_to_bf16(x) if bf16 else x
    return fn


def _normal(mu: float, sigma: float, bf16: bool):
    def fn(rng, count):
        x = rng.standard_normal(count, dtype=np.float32)
        if sigma != 1.0:
            x *= np.float32(sigma)
        if mu != 0.0:
            x += np.float32(mu)
        return f32_to_bf16(x) if bf16 else x
    return fn


def _neg_softplus_clamped(mu: float, sigma: float):
    def fn(rng, count):
        x = rng.standard_normal(count, dtype=np.float32) * np.float32(sigma) + np.float32(mu)
        # -softplus(x) = -(max(x,0) + log1p(exp(-|x|)))
        y = -(np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x))))
        return np.clip(y, -5.0, 0.0).astype(np.float32)
    return fn


def _sigmoid(rng, count):
    x = rng.standard_normal(count, dtype=np.float32)
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


@dataclass
class KDAInputs:
    """One seeded workload: host arrays plus shape metadata."""
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    bf16: bool
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    beta: np.ndarray
    initial_state: np.ndarray | None
    cu_seqlens: np.ndarray | None
    extra: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else len(self.cu_seqlens) - 1

    @property
    def tokens(self) -> int:
        """Total tokens over all sequences (each counted once, not per head)."""
        return self.B * self.T

    @property
    def seq_lens(self) -> np.ndarray:
        if self.cu_seqlens is None:
            return np.full(self.B, self.T, dtype=np.int64)
        return np.diff(self.cu_seqlens.astype(np.int64))


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, *, bf16: bool = True, seed: int = 0,
                chunk: int = 64, gate_mu: float = 0.0, gate_sigma: float = 1.0,
                state_sigma: float | None = None, seq_lens=None, pin_frac: float = 0.0,
                name: str = "custom") -> KDAInputs:
    """General seeded generator.

    ``seq_lens`` (list of ints) packs sequences along T with B=1 (cu_seqlens);
    otherwise B sequences of length T.  ``state_sigma`` None gives a zero (absent)
    initial state.  ``pin_frac`` pins that share of (head, channel) pairs to
    log_alpha = -5 and another disjoint share to 0.
    """
    ss = np.random.SeedSequence(seed)
    kq, kk, kv, kb, ka, ks, kl, kp = ss.spawn(8)
    if seq_lens is not None:
        seq_lens = [int(x) for x in seq_lens]
        B, T = 1, int(sum(seq_lens))
        cu = np.zeros(len(seq_lens) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(seq_lens)
    else:
        cu = None
    n_seq = B if cu is None else len(cu) - 1
    qk_dtype = np.uint16 if bf16 else np.float32
    q = np.empty((B, T, H, dk), dtype=qk_dtype)
    k = np.empty((B, T, H, dk), dtype=qk_dtype)
    v = np.empty((B, T, H, dv), dtype=qk_dtype)
    la = np.empty((B, T, H, dk), dtype=np.float32)
    be = np.empty((B, T, H), dtype=np.float32)
    _blocked(kq, q.size, dk, _unit_rows(dk, bf16), q)
    _blocked(kk, k.size, dk, _unit_rows(dk, bf16), k)
    _blocked(kv, v.size, dv, _normal(0.0, 1.0, bf16), v)
    _blocked(kb, be.size, 1, _sigmoid, be)
    _blocked(ka, la.size, dk, _neg_softplus_clamped(gate_mu, gate_sigma), la)
    s0 = None
    if state_sigma is not None:
        s0 = np.empty((n_seq, H, dk, dv), dtype=np.float32)
        _blocked(ks, s0.size, dv, _normal(0.0, state_sigma, False), s0)
    extra = {}
    if pin_frac > 0:
        n_pairs = H * dk
        n_pin = int(round(pin_frac * n_pairs))
        perm = np.random.default_rng(kp).permutation(n_pairs)
        floor_pairs, one_pairs = perm[:n_pin], perm[n_pin:2 * n_pin]
        la2 = la.reshape(B * T, H * dk)
        la2[:, floor_pairs] = -5.0
        la2[:, one_pairs] = 0.0
        extra["pinned_floor"] = floor_pairs
        extra["pinned_one"] = one_pairs
    if cu is not None:
        q, k, v, la, be = (x.reshape((T,) + x.shape[2:]) for x in (q, k, v, la, be))
    return KDAInputs(name=name, B=B, T=T, H=H, dk=dk, dv=dv, chunk=chunk, bf16=bf16, q=q, k=k, v=v,
                     log_alpha=la, beta=be, initial_state=s0, cu_seqlens=cu, extra=extra)


def packed_lengths(n: int, lo: int, hi: int, seed: int = 0) -> list[int]:
    """Sequence lengths uniform on the closed range [lo, hi] (integers)."""
    kl = np.random.SeedSequence(seed).spawn(8)[6]
    return [int(x) for x in np.random.default_rng(kl).integers(lo, hi + 1, size=n)]


WORKLOADS = {
    "tiny_fp32": dict(B=1, T=256, H=1, dk=64, dv=64, bf16=False, gate_mu=0.0, gate_sigma=1.0,
                      state_sigma=None),
    "b2_t4k": dict(B=2, T=4096, H=8, dk=128, dv=128, bf16=True, gate_mu=0.0, gate_sigma=2.0,
                   state_sigma=0.02),
    "prefill_64k": dict(B=1, T=65536, H=32, dk=128, dv=128, bf16=True, gate_mu=0.0,
                        gate_sigma=1.0, state_sigma=None, pin_frac=0.10),
    "packed_16": dict(B=1, T=None, H=16, dk=128, dv=128, bf16=True, gate_mu=0.0, gate_sigma=2.0,
                      state_sigma=0.02, packed=(16, 1024, 32768)),
    "prefill_1m": dict(B=1, T=1 << 20, H=8, dk=128, dv=128, bf16=True, gate_mu=-1.0,
                       gate_sigma=1.0, state_sigma=None),
    # decode / multi-token verify steps on resident states (kda_decode): B
    # sequences of T new tokens each; the states (B x 8 heads x 64 KiB) are
    # larger than the 126 MB L2.
    "decode_1024x1": dict(B=1024, T=1, H=8, dk=128, dv=128, bf16=True, gate_mu=-1.0,
                          gate_sigma=1.0, state_sigma=0.3, step="decode"),
    "verify_512x4": dict(B=512, T=4, H=8, dk=128, dv=128, bf16=True, gate_mu=-1.0,
                         gate_sigma=1.0, state_sigma=0.3, step="decode"),
}


def is_decode(name: str) -> bool:
    """True for the workloads that time a decode / verify step (kda_decode)."""
    return WORKLOADS[name].get("step") == "decode"


def workload(name: str, seed: int = 0) -> KDAInputs:
    """Build one of the five named workloads (see the module docstring)."""
    spec = dict(WORKLOADS[name])
    spec.pop("step", None)
    packed = spec.pop("packed", None)
    if packed is not None:
        lens = packed_lengths(*packed, seed=seed)
        spec.pop("T")
        return make_inputs(T=0, seq_lens=lens, seed=seed, name=name, **spec)
    return make_inputs(seed=seed, name=name, **spec)


def algorithmic_bytes(inp: KDAInputs) -> int:
    """Bytes one forward call must move at minimum: every input read once, every
    output written once (q, k, v, log_alpha, beta, out; states when present)."""
    e = 2 if inp.bf16 else 4
    th = inp.tokens * inp.H
    b = th * (2 * inp.dk * e + inp.dv * e + inp.dk * 4 + 4 + inp.dv * e)
    st = inp.n_seqs * inp.H * inp.dk * inp.dv * 4
    b += st  # final state written
    if inp.initial_state is not None:
        b += st
    return b


def algorithmic_flops(inp: KDAInputs, chunk: int = 64) -> float:
    """Chunkwise FLOPs per call with triangular products counted as triangles.

    Per full chunk of C tokens and one head: A = strict-lower(K~ K^T) C(C-1)/2*dk
    MACs; the triangular solve ~C^3/6; W, U', P, P.U each C(C+1)/2 * width; and
    the three state products W.S, Q~.S, K^T.U each C*dk*dv MACs.
    """
    C, dk, dv = chunk, inp.dk, inp.dv
    tri = C * (C + 1) / 2
    macs = (C * (C - 1) / 2) * dk + C ** 3 / 6 + tri * dk + tri * dv + tri * dk + tri * dv \
        + 3 * C * dk * dv
    per_token = 2.0 * macs / C
    return per_token * inp.tokens * inp.H


__all__ = ["KDAInputs", "make_inputs", "workload", "WORKLOADS", "is_decode", "f32_to_bf16", "bf16_to_f32",
           "packed_lengths", "algorithmic_bytes", "algorithmic_flops"]
