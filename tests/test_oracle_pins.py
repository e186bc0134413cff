"""Pins for the fp64 oracle: each check ties it to something other than itself.

Sources of truth (no page prints a worked example, so every pin is a closed
form, a brute-force loop written independently here, a special case or an
invariant the pages state):
  * RetNet "Key Innovation": D[n,m] = gamma^(n-m), parallel == recurrent.
  * RetNet "Triple Paradigm": parallel, recurrent and chunkwise agree.
  * RetNet "Multi-Scale Retention": gamma_h = 1 - 2^(-5-h).
  * mLSTM "Core idea" (DeepChrInteract-v2): C_t = f C + i v (x) k, gates
    stabilised in log space (the stabiliser must not change h).
  * xLSTM 7B "Modelled costs": 64.1 MiB of state at 128K tokens.
"""
import math

import numpy as np
import pytest

import oracle


def rand_case(rng, B=2, NH=3, S=13, DHQK=6, DHV=4, nb=1, with_state=False, with_o=False,
              f_mean=0.5):
    q = rng.standard_normal((B, NH, S, DHQK))
    k = rng.standard_normal((B, NH, S, DHQK)) / math.sqrt(DHQK)
    v = rng.standard_normal((B, NH, S, DHV))
    ig = rng.standard_normal((B, NH, S))
    fg = rng.standard_normal((B, NH, S)) + f_mean
    kw = dict(igate=ig, fgate=fg, num_blocks=nb)
    if with_o:
        kw["ogate"] = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, NH, S, DHV))))
    if with_state:
        dk, dv = DHQK // nb, DHV // nb
        kw["C0"] = rng.standard_normal((B, NH, nb, dv, dk)) * 0.3
        kw["n0"] = rng.standard_normal((B, NH, nb, dk)) * 0.3
        kw["m0"] = rng.standard_normal((B, NH))
    return q, k, v, kw


def relerr(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- 1. parallel form
@pytest.mark.parametrize("nb,with_state,with_o,shape", [
    (1, False, False, (2, 3, 13, 6, 4)),
    (1, True, True, (1, 2, 17, 5, 7)),
    (2, True, False, (2, 2, 11, 8, 6)),
    (4, False, True, (1, 3, 9, 8, 12)),
])
def test_sequential_equals_quadratic_parallel_form(nb, with_state, with_o, shape):
    rng = np.random.default_rng(1)
    B, NH, S, DHQK, DHV = shape
    q, k, v, kw = rand_case(rng, B, NH, S, DHQK, DHV, nb, with_state, with_o)
    hs, Cs, ns, ms = oracle.sequential(q, k, v, **kw)
    hp, Cp, np_, mp = oracle.parallel_form(q, k, v, **kw)
    assert relerr(hs, hp) < 1e-12
    assert relerr(Cs, Cp) < 1e-12
    assert relerr(ns, np_) < 1e-12
    assert np.max(np.abs(ms - mp)) < 1e-12


@pytest.mark.parametrize("with_state", [False, True])
def test_retention_sequential_equals_parallel_form(with_state):
    rng = np.random.default_rng(2)
    q, k, v, kw = rand_case(rng, 2, 4, 19, 6, 5, 1, with_state)
    kw = {"C0": kw["C0"]} if with_state else {}
    hs, Cs, _, _ = oracle.sequential(q, k, v, retention=True, **kw)
    hp, Cp, _, _ = oracle.parallel_form(q, k, v, retention=True, **kw)
    assert relerr(hs, hp) < 1e-12
    assert relerr(Cs, Cp) < 1e-12


# ---------------------------------------------------------------- 2. retention closed forms
def test_retention_gamma_values():
    g = oracle.retention_gamma(8)
    assert g[0] == 0.96875 and g[7] == 1.0 - 2.0 ** -12
    assert np.all(g == 1.0 - 2.0 ** (-5.0 - np.arange(8)))


@pytest.mark.parametrize("NH", [1, 4])
def test_retention_geometric_series_closed_form(NH):
    # dk = dv = 1, q = k = v = 1: h_t = sum_{s<=t} gamma^(t-s) = (1 - gamma^t) / (1 - gamma)
    S = 50
    ones = np.ones((1, NH, S, 1))
    h, C, _, _ = oracle.sequential(ones, ones, ones, retention=True)
    for hd in range(NH):
        g = 1.0 - 2.0 ** (-5 - hd)
        t = np.arange(1, S + 1)
        expect = (1.0 - g ** t) / (1.0 - g)
        assert np.max(np.abs(h[0, hd, :, 0] - expect) / expect) < 1e-13
        assert abs(C[0, hd, 0, 0, 0] - expect[-1]) / expect[-1] < 1e-13


def test_retention_page_orientation_brute_force():
    # The page's recurrent form keeps s = sum K^T V ([dk, dv]) and reads o = Q s.
    # Written here as a direct double loop in that orientation; the oracle keeps
    # C = s^T ([dv, dk]).  dk != dv so a transposed operand cannot pass.
    rng = np.random.default_rng(3)
    B, NH, S, dk, dv = 1, 3, 9, 3, 5
    q = rng.standard_normal((B, NH, S, dk))
    k = rng.standard_normal((B, NH, S, dk))
    v = rng.standard_normal((B, NH, S, dv))
    h, C, _, _ = oracle.sequential(q, k, v, retention=True)
    for hd in range(NH):
        gamma = 1.0 - 2.0 ** (-5 - hd)
        s = np.zeros((dk, dv))
        for t in range(S):
            for a in range(dk):
                for b in range(dv):
                    s[a, b] = gamma * s[a, b] + k[0, hd, t, a] * v[0, hd, t, b]
            o = np.zeros(dv)
            for b in range(dv):
                for a in range(dk):
                    o[b] += q[0, hd, t, a] * s[a, b]
            assert np.allclose(h[0, hd, t], o, rtol=1e-13, atol=1e-13)
        assert np.allclose(C[0, hd, 0], s.T, rtol=1e-13, atol=1e-13)


def test_retention_decay_matrix_closed_form():
    # Y = (Q K^T * D) V with D[n, m] = gamma^(n-m) for n >= m, else 0, built entry by entry.
    rng = np.random.default_rng(4)
    B, NH, S, dk, dv = 1, 2, 12, 4, 3
    q = rng.standard_normal((B, NH, S, dk))
    k = rng.standard_normal((B, NH, S, dk))
    v = rng.standard_normal((B, NH, S, dv))
    h, _, _, _ = oracle.sequential(q, k, v, retention=True)
    for hd in range(NH):
        gamma = 1.0 - 2.0 ** (-5 - hd)
        D = np.zeros((S, S))
        for n_ in range(S):
            for m_ in range(S):
                D[n_, m_] = gamma ** (n_ - m_) if n_ >= m_ else 0.0
        Y = (q[0, hd] @ k[0, hd].T * D) @ v[0, hd]
        assert relerr(h[0, hd], Y) < 1e-13


def test_retention_block_diagonal_uses_head_gamma():
    # num_blocks = 2: each block is its own retention memory over its slice of q, k, v,
    # decayed by the gamma of the head it belongs to (closed-form D per block).
    rng = np.random.default_rng(14)
    B, NH, S, DHQK, DHV, nb = 1, 3, 10, 6, 4, 2
    q = rng.standard_normal((B, NH, S, DHQK))
    k = rng.standard_normal((B, NH, S, DHQK))
    v = rng.standard_normal((B, NH, S, DHV))
    h, _, _, _ = oracle.sequential(q, k, v, retention=True, num_blocks=nb)
    dk, dv = DHQK // nb, DHV // nb
    for hd in range(NH):
        gamma = 1.0 - 2.0 ** (-5 - hd)
        D = np.array([[gamma ** (a - b) if a >= b else 0.0 for b in range(S)] for a in range(S)])
        for j in range(nb):
            Q = q[0, hd, :, j * dk:(j + 1) * dk]
            K = k[0, hd, :, j * dk:(j + 1) * dk]
            V = v[0, hd, :, j * dv:(j + 1) * dv]
            assert relerr(h[0, hd, :, j * dv:(j + 1) * dv], (Q @ K.T * D) @ V) < 1e-13


# ---------------------------------------------------------------- 3. hand-derived example
def test_hand_derived_two_steps():
    # dk = dv = 1, q = k = v = 1, itilde = -1, ftilde = 0 (log f = -ln 2), zero state.
    # t=1: m = max(-ln2 + 0, -1) = -ln2; f' = 1; i' = e^{-1+ln2} = 2/e; C' = n' = 2/e;
    #      h = (2/e) / max(2/e, e^{ln2} = 2) = 1/e.
    # t=2: m = max(-2 ln2, -1) = -1; f' = e^{-ln2 - ln2 + 1} = e/4; i' = 1;
    #      C' = n' = (e/4)(2/e) + 1 = 1.5;  h = 1.5 / max(1.5, e) = 1.5/e.
    one = np.ones((1, 1, 2, 1))
    ig = np.full((1, 1, 2), -1.0)
    fg = np.zeros((1, 1, 2))
    h, C, n, m = oracle.sequential(one, one, one, igate=ig, fgate=fg)
    assert abs(h[0, 0, 0, 0] - math.exp(-1)) < 1e-15
    assert abs(h[0, 0, 1, 0] - 1.5 * math.exp(-1)) < 1e-15
    assert abs(m[0, 0] - (-1.0)) < 1e-15
    assert abs(C[0, 0, 0, 0, 0] - 1.5) < 1e-15 and abs(n[0, 0, 0, 0] - 1.5) < 1e-15
    # unstabilised check: C_2 = f2 (i1 v k) + i2 v k = 0.5 e^{-1} + e^{-1} = 1.5 e^{-1} = C' e^{m}
    assert abs(C[0, 0, 0, 0, 0] * math.exp(m[0, 0]) - 1.5 * math.exp(-1)) < 1e-15
    # with itilde = 0 every output is exactly 1
    h0, _, _, _ = oracle.sequential(one, one, one, igate=np.zeros((1, 1, 2)), fgate=fg)
    assert np.all(np.abs(h0 - 1.0) < 1e-15)


# ---------------------------------------------------------------- 4. f = 1, i = 1
def test_unit_gates_reduce_to_floored_causal_linear_attention():
    # ftilde = 40 -> f = 1 - 4e-18 (1 in fp64), itilde = 0 -> i = 1, m = 0 throughout:
    # h_t = sum_{s<=t} (q_t.k_s) v_s / max(|sum_{s<=t} q_t.k_s|, 1)
    rng = np.random.default_rng(5)
    B, NH, S, dk, dv = 1, 2, 10, 3, 4
    q = rng.standard_normal((B, NH, S, dk))
    k = rng.standard_normal((B, NH, S, dk))
    v = rng.standard_normal((B, NH, S, dv))
    h, _, _, m = oracle.sequential(q, k, v, igate=np.zeros((B, NH, S)),
                                   fgate=np.full((B, NH, S), 40.0))
    assert np.all(m == 0.0)
    for hd in range(NH):
        for t in range(S):
            num = np.zeros(dv)
            den = 0.0
            for s in range(t + 1):
                a = float(np.dot(q[0, hd, t], k[0, hd, s]))
                num += a * v[0, hd, s]
                den += a
            assert np.allclose(h[0, hd, t], num / max(abs(den), 1.0), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- 5. stabiliser invariance
@pytest.mark.parametrize("nb,with_o", [(1, False), (2, True)])
def test_stabiliser_does_not_change_h(nb, with_o):
    rng = np.random.default_rng(6)
    B, NH, S, DHQK, DHV = 2, 2, 40, 8, 6
    q, k, v, kw = rand_case(rng, B, NH, S, DHQK, DHV, nb, False, with_o, f_mean=2.0)
    hs, Cs, ns, ms = oracle.sequential(q, k, v, **kw)
    hu, Cu, nu = oracle.unstabilised(q, k, v, kw["igate"], kw["fgate"], kw.get("ogate"),
                                     num_blocks=nb)
    assert relerr(hs, hu) < 1e-11
    scale = np.exp(ms)[:, :, None, None, None]
    assert relerr(Cs * scale, Cu) < 1e-11
    assert relerr(ns * np.exp(ms)[:, :, None, None], nu) < 1e-11


def test_stabiliser_keeps_large_gates_finite():
    # itilde = 200 would overflow exp() in the raw form; the stabilised recurrence stays finite
    rng = np.random.default_rng(7)
    q, k, v, kw = rand_case(rng, 1, 1, 16, 4, 4)
    kw["igate"] = kw["igate"] + 200.0
    h, C, n, m = oracle.sequential(q, k, v, **kw)
    assert np.all(np.isfinite(h)) and np.all(np.isfinite(C)) and m[0, 0] > 190


# ---------------------------------------------------------------- 6. cross-mode invariants
@pytest.mark.parametrize("retention", [False, True])
@pytest.mark.parametrize("chunk", [1, 2, 4, 5, 8, 16, 32])
def test_chunkwise_equals_sequential(chunk, retention):
    rng = np.random.default_rng(8)
    q, k, v, kw = rand_case(rng, 1, 3, 32, 6, 5, 1, True, not retention)
    if retention:
        kw = {"C0": kw["C0"]}
    hs, Cs, ns, ms = oracle.sequential(q, k, v, retention=retention, **kw)
    hc, Cc, nc, mc = oracle.chunkwise(q, k, v, retention=retention, chunk=chunk, **kw)
    assert relerr(hs, hc) < 1e-11
    assert relerr(Cs, Cc) < 1e-11
    if not retention:
        assert relerr(ns, nc) < 1e-11
        assert np.max(np.abs(ms - mc)) < 1e-12


def test_split_and_resume_equals_one_pass():
    rng = np.random.default_rng(9)
    q, k, v, kw = rand_case(rng, 2, 2, 30, 6, 4, 2, True, True)
    h, C, n, m = oracle.sequential(q, k, v, **kw)
    cut = 11
    first = {key: (val[:, :, :cut] if key in ("igate", "fgate", "ogate") else val)
             for key, val in kw.items()}
    h1, C1, n1, m1 = oracle.sequential(q[:, :, :cut], k[:, :, :cut], v[:, :, :cut], **first)
    second = {key: val[:, :, cut:] for key, val in kw.items() if key in ("igate", "fgate", "ogate")}
    h2, C2, n2, m2 = oracle.sequential(q[:, :, cut:], k[:, :, cut:], v[:, :, cut:],
                                       C0=C1, n0=n1, m0=m1, num_blocks=2, **second)
    assert relerr(np.concatenate([h1, h2], axis=2), h) < 1e-13
    assert relerr(C2, C) < 1e-13 and relerr(n2, n) < 1e-13 and np.max(np.abs(m2 - m)) < 1e-14


def test_token_by_token_steps_equal_one_pass():
    rng = np.random.default_rng(10)
    q, k, v, kw = rand_case(rng, 2, 2, 7, 4, 6, 1, True)
    h, C, n, m = oracle.sequential(q, k, v, **kw)
    Ct, nt, mt = kw["C0"], kw["n0"], kw["m0"]
    for t in range(7):
        ht, Ct, nt, mt = oracle.sequential(q[:, :, t:t + 1], k[:, :, t:t + 1], v[:, :, t:t + 1],
                                           igate=kw["igate"][:, :, t:t + 1],
                                           fgate=kw["fgate"][:, :, t:t + 1], C0=Ct, n0=nt, m0=mt)
        assert relerr(ht[:, :, 0], h[:, :, t]) < 1e-13
    assert relerr(Ct, C) < 1e-13 and np.max(np.abs(mt - m)) < 1e-14


# ---------------------------------------------------------------- 7. block-diagonal memory
def test_block_diagonal_equals_independent_subheads():
    # num_blocks = nb is nb independent memories per head sharing the head's gates
    rng = np.random.default_rng(11)
    B, NH, S, DHQK, DHV, nb = 2, 2, 12, 8, 6, 2
    q, k, v, kw = rand_case(rng, B, NH, S, DHQK, DHV, nb, True)
    h, C, n, m = oracle.sequential(q, k, v, **kw)
    dk, dv = DHQK // nb, DHV // nb

    def sub(x, d):  # [B,NH,S,nb*d] -> [B,NH*nb,S,d]
        return x.reshape(B, NH, S, nb, d).transpose(0, 1, 3, 2, 4).reshape(B, NH * nb, S, d)

    rep = lambda g: np.repeat(g, nb, axis=1)
    hs, Cs, ns, ms = oracle.sequential(
        sub(q, dk), sub(k, dk), sub(v, dv), igate=rep(kw["igate"]), fgate=rep(kw["fgate"]),
        C0=kw["C0"].reshape(B, NH * nb, 1, dv, dk), n0=kw["n0"].reshape(B, NH * nb, 1, dk),
        m0=rep(kw["m0"]))
    back = hs.reshape(B, NH, nb, S, dv).transpose(0, 1, 3, 2, 4).reshape(B, NH, S, DHV)
    assert np.array_equal(back, h)
    assert np.array_equal(Cs.reshape(C.shape), C)
    assert np.array_equal(ms[:, ::nb], m)


# ---------------------------------------------------------------- 8. linearity in v
def test_h_is_linear_in_v():
    rng = np.random.default_rng(12)
    q, k, v, kw = rand_case(rng, 1, 2, 15, 5, 3, 1, False, True)
    h1, C1, n1, m1 = oracle.sequential(q, k, v, **kw)
    h2, C2, n2, m2 = oracle.sequential(q, k, 2.0 * v, **kw)
    assert np.array_equal(h2, 2.0 * h1) and np.array_equal(C2, 2.0 * C1)
    assert np.array_equal(n2, n1) and np.array_equal(m2, m1)


# ---------------------------------------------------------------- 9. state size
def test_state_size_matches_modelled_cost():
    # xLSTM 7B: 32 layers x 8 heads, qk 256 x v 512 per head, BF16 -> "64.1 MiB"
    b = oracle.state_bytes(32, 8, 256, 512, 2)
    assert b == 67_240_448
    assert round(b / 2 ** 20, 1) == 64.1


def test_state_does_not_grow_with_sequence_length():
    rng = np.random.default_rng(13)
    shapes = set()
    for S in (1, 5, 40):
        q, k, v, kw = rand_case(rng, 1, 2, S, 4, 4)
        _, C, n, m = oracle.sequential(q, k, v, **kw)
        shapes.add((C.shape, n.shape, m.shape))
    assert len(shapes) == 1
