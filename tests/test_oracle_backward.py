"""Pins for the fp64 backward oracle: central finite differences of the forward oracle.

The loss is L = sum_t h_t . W_t + <U, exp(m_S) C'_S> + u . exp(m_S) n'_S: a linear functional
of h and of the final state in unstabilised units, which is smooth in every input (the
stabiliser m cancels; mLSTM "Core idea", gates stabilised in log space).  Its gradient in
stabilised units with m_S held fixed is dC = exp(m_S) U, dn = exp(m_S) u.  Each analytic
gradient of ``oracle.sequential_backward`` is compared with (L(x+e) - L(x-e)) / 2e computed
with ``oracle.sequential`` (the C recurrence), element by element.
"""
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import rand_case


def _loss(q, k, v, kw, W, U, u, retention):
    h, C, n, m = oracle.sequential(q, k, v, retention=retention, **kw)
    L = float(np.sum(h * W))
    if retention:
        return L + float(np.sum(U * C))
    sc = np.exp(m)[:, :, None, None]
    return L + float(np.sum(U * C * sc[..., None])) + float(np.sum(u * n * sc))


def _fd_check(q, k, v, kw, retention, rng, eps=1e-6):
    B, NH, S, _ = q.shape
    nb = kw.get("num_blocks", 1)
    W = rng.standard_normal(q.shape[:3] + (v.shape[-1],))
    dkk, dvv = q.shape[-1] // nb, v.shape[-1] // nb
    U = rng.standard_normal((B, NH, nb, dvv, dkk)) * 0.5
    u = rng.standard_normal((B, NH, nb, dkk)) * 0.5
    h, C, n, m = oracle.sequential(q, k, v, retention=retention, **kw)
    if retention:
        dC, dn = U, None
    else:
        sc = np.exp(m)[:, :, None, None]
        dC, dn = U * sc[..., None], u * sc
    g = oracle.sequential_backward(q, k, v, W, retention=retention, dC=dC, dn=dn, **kw)
    named = {"q": (q, "dq"), "k": (k, "dk"), "v": (v, "dv")}
    for key, grad in (("igate", "di"), ("fgate", "df"), ("ogate", "do"), ("C0", "dC0"), ("n0", "dn0"),
                      ("m0", "dm0")):
        if key in kw and g[grad] is not None:
            named[key] = (kw[key], grad)
    checked = 0
    for key, (x, grad) in named.items():
        x = np.array(x, dtype=np.float64)
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            if key in ("q", "k", "v"):
                args = {"q": q, "k": k, "v": v}
                args[key] = xp
                lp = _loss(args["q"], args["k"], args["v"], kw, W, U, u, retention)
                args[key] = xm
                lm = _loss(args["q"], args["k"], args["v"], kw, W, U, u, retention)
            else:
                kp, km = dict(kw), dict(kw)
                kp[key], km[key] = xp, xm
                lp = _loss(q, k, v, kp, W, U, u, retention)
                lm = _loss(q, k, v, km, W, U, u, retention)
            fd[idx] = (lp - lm) / (2 * eps)
        an = g[grad]
        scale = max(np.max(np.abs(fd)), 1e-12)
        err = np.max(np.abs(an - fd)) / scale
        assert err < 1e-6, (key, err)
        checked += 1
    return checked, g


def test_backward_matches_finite_differences_mlstm_with_state_and_ogate():
    rng = np.random.default_rng(11)
    q, k, v, kw = rand_case(rng, 1, 2, 7, 4, 3, 1, with_state=True, with_o=True)
    checked, _ = _fd_check(q, k, v, kw, False, rng)
    assert checked == 9


def test_backward_matches_finite_differences_block_diagonal():
    rng = np.random.default_rng(12)
    q, k, v, kw = rand_case(rng, 1, 2, 6, 4, 6, 2, with_state=True, with_o=False)
    _fd_check(q, k, v, kw, False, rng)


def test_backward_matches_finite_differences_retention():
    rng = np.random.default_rng(13)
    q, k, v, kw = rand_case(rng, 1, 3, 6, 3, 2, 1, with_state=True)
    kw = {"C0": kw["C0"]}
    checked, g = _fd_check(q, k, v, kw, True, rng)
    assert checked == 4 and g["di"] is None and g["df"] is None


@pytest.mark.parametrize("big", [False, True])
def test_backward_both_denominator_branches(big):
    # small q, k: |n . q| below the floor exp(-m) for most tokens; large: above it
    rng = np.random.default_rng(14 + big)
    q, k, v, kw = rand_case(rng, 1, 1, 8, 4, 3, 1)
    s = 6.0 if big else 0.05
    _fd_check(q * s, k * s, v, kw, False, rng)


def test_backward_is_linear_in_dh():
    rng = np.random.default_rng(15)
    q, k, v, kw = rand_case(rng, 1, 2, 5, 4, 3, 1, with_state=True)
    dh = rng.standard_normal(q.shape[:3] + (3,))
    g1 = oracle.sequential_backward(q, k, v, dh, **kw)
    g2 = oracle.sequential_backward(q, k, v, 2.0 * dh, **kw)
    for key in ("dq", "dk", "dv", "di", "df", "dC0", "dn0", "dm0"):
        assert np.max(np.abs(g2[key] - 2.0 * g1[key])) <= 1e-12 * max(1.0, np.max(np.abs(g1[key])))
