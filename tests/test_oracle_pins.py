"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test targets a plausible mistake: a transposed state (rows are key
channels), decay applied after instead of before the erase, the output reading
the old state, a wrong sign on the erase, a dropped clamp, a broken chunkwise
rewrite.  Shapes use d_k != d_v so that a transposed operand cannot pass.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs, f32_to_bf16, bf16_to_f32

RNG = np.random.default_rng(1234)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(T, H, dk, dv, *, s0=True, seed=0):
    x = make_inputs(1, T, H, dk, dv, bf16=False, seed=seed, state_sigma=0.3 if s0 else None)
    return x


def _rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ---------------------------------------------------------------- closed forms
def test_single_token_from_zero_state():
    """T=1, S0=0: S = beta k v^T and o = beta (k.q) v (the output sees the write)."""
    dk, dv = 5, 3
    q = RNG.standard_normal((1, 1, 1, dk)).astype(np.float32)
    k = RNG.standard_normal((1, 1, 1, dk)).astype(np.float32)
    v = RNG.standard_normal((1, 1, 1, dv)).astype(np.float32)
    la = np.full((1, 1, 1, dk), -0.7, np.float32)
    be = np.full((1, 1, 1), 0.37, np.float32)
    o, s = oracle.recurrent(q, k, v, la, be)
    kk, vv, qq, b = k[0, 0, 0].astype(float), v[0, 0, 0].astype(float), q[0, 0, 0].astype(float), 0.37
    b = float(np.float32(0.37))
    np.testing.assert_allclose(s[0, 0], b * np.outer(kk, vv), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(o[0, 0, 0], b * (kk @ qq) * vv, rtol=1e-14, atol=1e-15)


def test_beta_zero_is_pure_decay_of_rows():
    """beta=0: S_t = Diag(prod_{s<=t} alpha_s) S0 (rows = key channels), o_t = S_t^T q_t."""
    T, dk, dv = 9, 6, 4
    x = _case(T, 1, dk, dv)
    be = np.zeros_like(x.beta)
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, be, x.initial_state)
    la = np.clip(x.log_alpha[0, :, 0, :].astype(float), -5, 0)
    S0 = x.initial_state[0, 0].astype(float)
    for t in range(T):
        St = np.exp(la[: t + 1].sum(0))[:, None] * S0
        np.testing.assert_allclose(o[0, t, 0], St.T @ x.q[0, t, 0].astype(float), rtol=1e-12,
                                   atol=1e-14)
    np.testing.assert_allclose(s[0, 0], np.exp(la.sum(0))[:, None] * S0, rtol=1e-12, atol=1e-15)


def test_beta_zero_no_decay_leaves_state_unchanged():
    T, dk, dv = 7, 4, 6
    x = _case(T, 2, dk, dv)
    o, s = oracle.recurrent(x.q, x.k, x.v, np.zeros_like(x.log_alpha), np.zeros_like(x.beta),
                            x.initial_state)
    np.testing.assert_array_equal(s, x.initial_state.astype(float))


def test_basis_keys_rewrite_one_row():
    """Keys e_{i_t}: row i_t <- (1-beta) alpha*row + beta v; other rows only decay.

    A closed form that follows a row of S scalar by scalar; it separates
    decay-before-erase from decay-after-erase and rows from columns.
    """
    T, dk, dv = 12, 5, 3
    idx = RNG.integers(0, dk, size=T)
    k = np.zeros((1, T, 1, dk), np.float32)
    k[0, np.arange(T), 0, idx] = 1.0
    q = RNG.standard_normal((1, T, 1, dk)).astype(np.float32)
    v = RNG.standard_normal((1, T, 1, dv)).astype(np.float32)
    la = (-RNG.uniform(0, 2, size=(1, T, 1, dk))).astype(np.float32)
    be = RNG.uniform(0.05, 0.95, size=(1, T, 1)).astype(np.float32)
    S0 = RNG.standard_normal((1, 1, dk, dv)).astype(np.float32)
    o, s = oracle.recurrent(q, k, v, la, be, S0)
    S = S0[0, 0].astype(float).copy()
    for t in range(T):
        a = np.exp(la[0, t, 0].astype(float))
        i = idx[t]
        b = float(be[0, t, 0])
        new = a[:, None] * S
        new[i] = (1 - b) * a[i] * S[i] + b * v[0, t, 0].astype(float)
        S = new
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0].astype(float), rtol=1e-12,
                                   atol=1e-13)
    np.testing.assert_allclose(s[0, 0], S, rtol=1e-12, atol=1e-13)


def test_full_write_with_query_equal_key_returns_value():
    """beta=1, unit k, q_t = k_t: o_t = v_t for ANY alpha and any state.

    (I - k k^T) removes everything the decayed state held along k, so the state
    returns exactly the value just written.  Fails if the decay is applied after
    the erase, if the output reads S_{t-1}, or if the erase sign is wrong.
    """
    T, dk, dv = 10, 8, 5
    x = _case(T, 1, dk, dv, seed=3)
    k = x.k.copy()
    be = np.ones_like(x.beta)
    o, _ = oracle.recurrent(k, k, x.v, x.log_alpha, be, x.initial_state)
    kd = k.astype(float)
    assert np.allclose(np.linalg.norm(kd, axis=-1), 1.0, atol=1e-6)
    # unit to fp32 rounding: the retrieval is exact up to 1 - |k|^2
    np.testing.assert_allclose(o, x.v.astype(float), atol=2e-6 * 8)


def test_orthonormal_keys_retrieve_all_values():
    """alpha=1, beta=1, orthonormal keys: S_T^T k_j = v_j for every j (any S0)."""
    dk, dv, T = 8, 5, 6
    Qm, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    keys = Qm[:, :T].T.astype(np.float32)  # rows orthonormal to fp32 rounding
    k = keys[None, :, None, :].copy()
    v = RNG.standard_normal((1, T, 1, dv)).astype(np.float32)
    S0 = RNG.standard_normal((1, 1, dk, dv)).astype(np.float32)
    o, s = oracle.recurrent(k, k, v, np.zeros((1, T, 1, dk), np.float32),
                            np.ones((1, T, 1), np.float32), S0)
    ST = s[0, 0]
    for j in range(T):
        np.testing.assert_allclose(ST.T @ keys[j].astype(float), v[0, j, 0], atol=5e-6)


# ---------------------------------------------------------------- brute force
def _dense_unrolled(q, k, v, la, be, S0):
    """Transition matrices built explicitly: Phi_t = (I - b k k^T) Diag(alpha_t)."""
    T, dk = k.shape[0], k.shape[1]
    Phis = []
    for t in range(T):
        a = np.exp(np.clip(la[t], -5, 0))
        Phis.append((np.eye(dk) - be[t] * np.outer(k[t], k[t])) @ np.diag(a))
    outs = []
    for t in range(T):
        St = np.eye(dk)
        for s_ in range(t + 1):
            St = Phis[s_] @ St
        St = St @ S0
        for j in range(t + 1):
            P = np.eye(dk)
            for s_ in range(j + 1, t + 1):
                P = Phis[s_] @ P
            St = St + P @ (be[j] * np.outer(k[j], v[j]))
        outs.append(St)
    return np.array([outs[t].T @ q[t] for t in range(T)]), outs[-1]


@pytest.mark.parametrize("T,dk,dv", [(1, 3, 2), (5, 4, 3), (16, 6, 5)])
def test_dense_unrolling_brute_force(T, dk, dv):
    x = make_inputs(1, T, 1, dk, dv, bf16=False, seed=T, state_sigma=0.5, gate_sigma=2.0)
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    f = lambda a: a[0, :, 0].astype(float)
    o_ref, s_ref = _dense_unrolled(f(x.q), f(x.k), f(x.v), f(x.log_alpha),
                                   x.beta[0, :, 0].astype(float), x.initial_state[0, 0].astype(float))
    assert _rel(o[0, :, 0], o_ref) < 1e-12
    assert _rel(s[0, 0], s_ref) < 1e-12


def _parse_golden(path):
    sect, data = None, {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        if line.startswith("["):
            sect = line.strip("[]")
            data.setdefault(sect, {})
            continue
        key, val = (x.strip() for x in line.split("=", 1))
        rows = [[Fraction(t) for t in r.split()] for r in val.split(";")]
        data[sect][key] = rows
    return data


def test_golden_hand_worked_basis_example():
    g = _parse_golden(os.path.join(GOLDEN, "basis_keys_3x2.txt"))
    inp, exp = g["inputs"], g["expected"]
    T = len(inp["k"])
    arr = lambda rows: np.array([[float(x) for x in r] for r in rows], np.float32)
    k = arr(inp["k"])[None, :, None, :]
    q = arr(inp["q"])[None, :, None, :]
    v = arr(inp["v"])[None, :, None, :]
    be = arr(inp["beta"])[0][None, :, None]
    la = np.zeros_like(k)
    S0 = arr(inp["S0"])[None, None]
    o, s = oracle.recurrent(q, k, v, la, be, S0)
    np.testing.assert_array_equal(o[0, :, 0], arr(exp["o"]).astype(float))
    np.testing.assert_array_equal(s[0, 0], arr(exp["S_final"]).astype(float))


# ---------------------------------------------------------------- clamp
def test_clamp_to_closed_interval():
    """log alpha outside [-5, 0] behaves exactly as its clamp; -5 and 0 are kept."""
    T, dk, dv = 20, 6, 4
    x = _case(T, 2, dk, dv, seed=5)
    wild = (RNG.standard_normal(x.log_alpha.shape) * 6).astype(np.float32)
    wild.reshape(-1)[:4] = [-5.0, 0.0, -5.0000005, 1e-3]
    o1, s1 = oracle.recurrent(x.q, x.k, x.v, wild, x.beta, x.initial_state)
    o2, s2 = oracle.recurrent(x.q, x.k, x.v, np.clip(wild, -5, 0), x.beta, x.initial_state)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)
    # the clamp value itself: beta=0 and log alpha=-9 decays by e^-5 per token
    z = np.zeros_like(x.beta)
    _, s3 = oracle.recurrent(x.q, x.k, x.v, np.full_like(wild, -9.0), z, x.initial_state)
    np.testing.assert_allclose(s3, np.exp(-5.0 * T) * x.initial_state.astype(float), rtol=1e-12)


# ---------------------------------------------------------------- chunkwise form
@pytest.mark.parametrize("chunk", [1, 2, 3, 16, 64, 128])
def test_chunked_form_matches_recurrence(chunk):
    x = make_inputs(2, 203, 2, 16, 12, bf16=False, seed=7, state_sigma=0.2, gate_sigma=2.0)
    o1, s1 = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    o2, s2 = oracle.chunked(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, chunk=chunk)
    assert _rel(o2, o1) < 1e-12
    assert _rel(s2, s1) < 1e-12


def test_chunked_form_at_clamp_floor():
    """All gates at -5 over 64-token chunks: exp(-+320) in the chunk form."""
    x = make_inputs(1, 300, 1, 32, 8, bf16=False, seed=8, state_sigma=0.2)
    la = np.full_like(x.log_alpha, -5.0)
    o1, s1 = oracle.recurrent(x.q, x.k, x.v, la, x.beta, x.initial_state)
    o2, s2 = oracle.chunked(x.q, x.k, x.v, la, x.beta, x.initial_state, chunk=64)
    assert _rel(o2, o1) < 1e-11
    assert np.abs(s2 - s1).max() < 1e-12


# ---------------------------------------------------------------- invariants
def test_packed_equals_separate_sequences():
    lens = [5, 0, 70, 1, 33]
    x = make_inputs(1, 0, 3, 8, 6, bf16=False, seed=9, seq_lens=lens, state_sigma=0.1)
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, x.cu_seqlens)
    cu = x.cu_seqlens
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        o_n, s_n = oracle.recurrent(x.q[None, sl], x.k[None, sl], x.v[None, sl],
                                    x.log_alpha[None, sl], x.beta[None, sl],
                                    x.initial_state[n:n + 1])
        np.testing.assert_array_equal(s[n], s_n[0])
        if L:
            np.testing.assert_array_equal(o[sl], o_n[0])
    # zero-length sequence: final state = initial state
    np.testing.assert_array_equal(s[1], x.initial_state[1].astype(float))


def test_resume_from_final_state():
    x = _case(150, 2, 8, 6, seed=10)
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    T1 = 61
    sl1, sl2 = slice(0, T1), slice(T1, None)
    cut = lambda a, sl: a[:, sl]
    o1, s1 = oracle.recurrent(cut(x.q, sl1), cut(x.k, sl1), cut(x.v, sl1), cut(x.log_alpha, sl1),
                              cut(x.beta, sl1), x.initial_state)
    o2, s2 = oracle.recurrent(cut(x.q, sl2), cut(x.k, sl2), cut(x.v, sl2), cut(x.log_alpha, sl2),
                              cut(x.beta, sl2), s1.astype(np.float32))
    np.testing.assert_array_equal(o1, o[:, sl1])
    # the state crosses the boundary as fp32, so the tail agrees to fp32 rounding
    assert _rel(o2, o[:, sl2]) < 1e-6
    assert _rel(s2, s) < 1e-6


def test_state_enters_affinely():
    """Output and final state are affine in S0: f(a+b) - f(0) = (f(a)-f(0)) + (f(b)-f(0)).

    a and b are multiples of 2^-10 so that a+b is exact in fp32.
    """
    # weak gates (log alpha ~ -0.05) so that S0 still matters after 40 tokens
    x = make_inputs(1, 40, 1, 6, 5, bf16=False, seed=11, state_sigma=0.3, gate_mu=-3.0)
    a = (np.round(x.initial_state * 1024) / 1024).astype(np.float32)
    b = (np.round(RNG.standard_normal(a.shape) * 300) / 1024).astype(np.float32)
    ab = a + b
    assert np.array_equal(ab.astype(np.float64), a.astype(np.float64) + b.astype(np.float64))
    f = lambda s0: oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, s0)
    (oa, sa), (ob, sb), (oab, sab), (o0, s0) = f(a), f(b), f(ab), f(np.zeros_like(a))
    assert _rel(oab - o0, (oa - o0) + (ob - o0)) < 1e-10
    assert _rel(sab - s0, (sa - s0) + (sb - s0)) < 1e-10


def test_bf16_bits_match_widened_fp32():
    x = make_inputs(1, 64, 2, 8, 8, bf16=True, seed=12)
    o1, s1 = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta)
    o2, s2 = oracle.recurrent(bf16_to_f32(x.q), bf16_to_f32(x.k), bf16_to_f32(x.v),
                              x.log_alpha, x.beta)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.5, 3.0e38], np.float32)
    r = bf16_to_f32(f32_to_bf16(vals))
    np.testing.assert_array_equal(r, np.array([1.0, 1.0, 1.0 + 2**-6, 1.0, -2.5,
                                               np.float32(2.9916e38)], np.float32)[:5].tolist()
                                  + [r[5]])
    assert abs(r[5] - 3.0e38) / 3.0e38 < 2**-8


# ---------------------------------------------------------------- output gate
# The gate that follows the attention passes a share of each output element on
# (aiblin.ru page, description of the layer stack).  Pins: it acts on the output
# only (never on the state), element by element, multiplicatively.
def test_gate_of_ones_is_the_ungated_output():
    x = _case(70, 2, 8, 6, seed=40)
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    og, sg = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state,
                              out_gate=np.ones_like(x.v))
    np.testing.assert_array_equal(o, og)
    np.testing.assert_array_equal(s, sg)


def test_gate_acts_on_one_element_only():
    """Zeroing the gate at one (token, head, channel) zeroes exactly that output
    element; other outputs and the final state are untouched, so the gate is
    outside the recurrence and indexed like the output (d_k != d_v)."""
    x = _case(50, 3, 8, 6, seed=41)
    g = np.ones_like(x.v)
    g[0, 17, 2, 4] = 0.0
    o, s = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    og, sg = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, out_gate=g)
    assert og[0, 17, 2, 4] == 0.0 and o[0, 17, 2, 4] != 0.0
    mask = np.ones(o.shape, bool)
    mask[0, 17, 2, 4] = False
    np.testing.assert_array_equal(og[mask], o[mask])
    np.testing.assert_array_equal(sg, s)


def test_gate_scales_each_output_exactly():
    """A power-of-two gate scales the output exactly; random gates act as the
    elementwise product (chunked form as well)."""
    x = _case(90, 2, 8, 6, seed=42)
    o, _ = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    og, _ = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state,
                             out_gate=np.full_like(x.v, 0.25))
    np.testing.assert_array_equal(og, 0.25 * o)
    g = RNG.uniform(0, 1, x.v.shape).astype(np.float32)
    oc, _ = oracle.chunked(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, chunk=16,
                           out_gate=g)
    assert _rel(oc, o * g.astype(np.float64)) < 1e-12


def test_gate_bf16_bits_match_widened_fp32():
    x = make_inputs(1, 40, 2, 8, 8, bf16=True, seed=43)
    g = f32_to_bf16(RNG.uniform(0, 1, (1, 40, 2, 8)).astype(np.float32))
    o1, _ = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, out_gate=g)
    o2, _ = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, out_gate=bf16_to_f32(g))
    np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------------- per-chunk operands
@pytest.mark.parametrize("chunk", [1, 8, 16, 64])
def test_chunk_operands_rebuild_the_recurrence(chunk):
    """The per-chunk operands, chained from a random state over a ragged sequence, give
    the token recurrence's outputs and final state; T inverts I + A."""
    x = make_inputs(1, 77, 2, 6, 5, bf16=False, seed=44, state_sigma=0.3, gate_sigma=2.0)
    o_ref, s_ref = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state)
    ops = oracle.chunk_operands(x.q, x.k, x.v, x.log_alpha, x.beta, chunk)
    n = ops["W"].shape[0]
    S = x.initial_state[0].astype(np.float64).copy()  # [H, dk, dv]
    outs = []
    for c in range(n):
        o_c = np.empty((chunk, 2, 5))
        for h in range(2):
            u = ops["U"][c, h] - ops["W"][c, h] @ S[h]
            o_c[:, h] = ops["Qt"][c, h] @ S[h] + ops["P"][c, h] @ u
            S[h] = ops["gamma"][c, h][:, None] * S[h] + ops["Kdec"][c, h].T @ u
            np.testing.assert_allclose((np.eye(chunk) + ops["A"][c, h]) @ ops["T"][c, h],
                                       np.eye(chunk), atol=1e-9)
        outs.append(o_c)
    o = np.concatenate(outs)[:77]
    assert _rel(o, o_ref.reshape(77, 2, 5)) < 1e-12
    assert _rel(S, s_ref[0]) < 1e-12


def test_chunk_operands_of_padding_rows_are_identity_steps():
    """Rows past a ragged end: zero W, U, P, Kdec rows, T's identity there, gamma from
    the last real token."""
    x = make_inputs(1, 20, 1, 4, 3, bf16=False, seed=45, gate_sigma=2.0)
    ops = oracle.chunk_operands(x.q, x.k, x.v, x.log_alpha, x.beta, 32)
    for name in ("W", "U", "Kdec", "Qt"):
        assert not ops[name][0, 0, 20:].any(), name
    assert not ops["P"][0, 0, 20:].any() and not ops["A"][0, 0, 20:].any()
    np.testing.assert_array_equal(ops["T"][0, 0, 20:, 20:], np.eye(12))
    g_last = np.cumsum(np.clip(x.log_alpha[0, :, 0].astype(np.float64), -5, 0), axis=0)[-1]
    np.testing.assert_allclose(ops["gamma"][0, 0], np.exp(g_last), rtol=1e-15)
