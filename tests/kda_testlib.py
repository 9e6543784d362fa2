"""Helpers shared by the GPU parity tests: device upload, comparison metrics."""
from __future__ import annotations

import numpy as np

# fp32 inputs: max |error| over all elements; bf16 inputs: relative Frobenius
# error per (sequence, head) over (tokens x d_v) for o and over (d_k x d_v) for
# the final state.
TOL_F32_MAX_ABS = 1e-4
TOL_BF16_REL_FRO = 2e-2
# bf16 inputs, per (sequence, head, 64-token chunk of the sequence): relative Frobenius
# error of o over the chunk's tokens x d_v, with the denominator floored at a quarter of
# the head's RMS over the same number of tokens (so a chunk whose outputs are near zero
# is judged against the head's scale).  The per-head bound averages over up to 2^20
# tokens; this one catches a single wrong chunk (a ragged tail, a segment boundary, a
# clamp-floor channel) that the average would hide.
TOL_BF16_REL_FRO_CHUNK = 4e-2


def to_device(inp, device="cuda"):
    import torch
    if inp.bf16:
        t = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(device)
    else:
        t = lambda a: torch.from_numpy(a).to(device)
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return dict(q=t(inp.q), k=t(inp.k), v=t(inp.v), log_alpha=f(inp.log_alpha), beta=f(inp.beta),
                initial_state=f(inp.initial_state), cu_seqlens=f(inp.cu_seqlens))


def out_to_f64(out):
    import torch
    return out.float().cpu().numpy().astype(np.float64) if out.dtype == torch.bfloat16 else \
        out.cpu().numpy().astype(np.float64)


def run_gpu(inp, **kw):
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    d = to_device(inp)
    d.update(kw)
    out, fs = kda_fwd(**d)
    torch.cuda.synchronize()
    return out_to_f64(out), fs.cpu().numpy().astype(np.float64)


def seq_bounds(inp):
    if inp.cu_seqlens is None:
        return [(n * inp.T, (n + 1) * inp.T) for n in range(inp.B)]
    cu = inp.cu_seqlens.astype(np.int64)
    return [(int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]


def rel_fro_per_head(o_gpu, o_ref, s_gpu, s_ref, inp, o_tokens=None):
    """Worst relative Frobenius error over (sequence, head) for o and final state."""
    H, dv = inp.H, inp.dv
    og = o_gpu.reshape(-1, H, dv)
    orf = o_ref.reshape(-1, H, dv)
    worst_o = 0.0
    for lo, hi in seq_bounds(inp):
        if o_tokens is not None:
            hi = min(hi, o_tokens)
        if hi <= lo:
            continue
        for h in range(H):
            ref = orf[lo:hi, h]
            den = np.linalg.norm(ref)
            err = np.linalg.norm(og[lo:hi, h] - ref)
            worst_o = max(worst_o, err / den if den > 0 else err)
    worst_s = 0.0
    for n in range(s_ref.shape[0]):
        for h in range(H):
            den = np.linalg.norm(s_ref[n, h])
            err = np.linalg.norm(s_gpu[n, h] - s_ref[n, h])
            worst_s = max(worst_s, err / den if den > 0 else err)
    return worst_o, worst_s


def rel_fro_per_chunk(o_gpu, o_ref, inp, o_tokens=None, chunk=64):
    """Worst per-chunk error of o (see TOL_BF16_REL_FRO_CHUNK) and where: (err, (seq, chunk, head))."""
    H, dv = inp.H, inp.dv
    og = o_gpu.reshape(-1, H, dv)
    orf = o_ref.reshape(-1, H, dv)
    worst, where = 0.0, None
    for n, (lo, hi) in enumerate(seq_bounds(inp)):
        if o_tokens is not None:
            hi = min(hi, o_tokens)
        if hi <= lo:
            continue
        L = hi - lo
        nc = (L + chunk - 1) // chunk
        pad = ((0, nc * chunk - L), (0, 0))
        dd = np.pad(((og[lo:hi] - orf[lo:hi]) ** 2).sum(-1), pad).reshape(nc, chunk, H).sum(1)
        rr = np.pad((orf[lo:hi] ** 2).sum(-1), pad).reshape(nc, chunk, H).sum(1)
        cnt = np.minimum(chunk, L - np.arange(nc) * chunk)[:, None]
        floor = 0.25 ** 2 * rr.sum(0, keepdims=True) / L * cnt
        e = np.sqrt(dd / np.maximum(np.maximum(rr, floor), 1e-300))
        i = np.unravel_index(int(np.argmax(e)), e.shape)
        if e[i] > worst:
            worst, where = float(e[i]), (n, int(i[0]), int(i[1]))
    return worst, where
