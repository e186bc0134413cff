"""Pins for the scalar-normaliser variant of the oracle (Edifice.Recurrent.XLSTMv2, "Key
Improvements" #2: n_t = f_t n_{t-1} + i_t, h_t = o_t (c_t / max(|n_t + bias|, 1))).

Each pin is independent of the oracle's stabilised recurrence: the raw (unstabilised)
recurrence written out here, a closed form of the scalar normaliser as a sum over the decay
matrix, and a hand-derived case with f = 1."""
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import rand_case, relerr


def raw_form(q, k, v, ig, fg, bias, og, C0, n0, m0, nb):
    """Unstabilised: C_t = f C + e^{itilde} v k^T with C_0 = e^{m0} C0', n likewise."""
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    dk, dv = DHQK // nb, DHV // nb
    h = np.zeros((B, NH, S, DHV))
    for b in range(B):
        for hd in range(NH):
            f = np.exp(oracle.log_sigmoid(fg[b, hd]))
            i = np.exp(ig[b, hd])
            n = math.exp(m0[b, hd]) * n0[b, hd]
            Cs = [math.exp(m0[b, hd]) * C0[b, hd, j] for j in range(nb)]
            for t in range(S):
                n = f[t] * n + i[t]
                den = max(abs(n + bias[hd]), 1.0)
                for j in range(nb):
                    sk, sv = slice(j * dk, (j + 1) * dk), slice(j * dv, (j + 1) * dv)
                    Cs[j] = f[t] * Cs[j] + i[t] * np.outer(v[b, hd, t, sv], k[b, hd, t, sk])
                    ht = Cs[j] @ q[b, hd, t, sk] / den
                    if og is not None:
                        ht = ht * og[b, hd, t, sv]
                    h[b, hd, t, sv] = ht
    return h


@pytest.mark.parametrize("nb,with_o", [(1, False), (2, True)])
def test_scalar_normaliser_equals_unstabilised_recurrence(nb, with_o):
    rng = np.random.default_rng(21)
    q, k, v, kw = rand_case(rng, 2, 2, 15, 4, 6, nb, with_state=True, with_o=with_o)
    n0 = rng.standard_normal((2, 2)) * 0.3
    bias = rng.standard_normal(2)
    h, C, n, m = oracle.sequential_scalar_normaliser(q, k, v, kw["igate"], kw["fgate"], bias, kw.get("ogate"),
                                                     kw["C0"], n0, kw["m0"], num_blocks=nb)
    hr = raw_form(q, k, v, kw["igate"], kw["fgate"], bias, kw.get("ogate"), kw["C0"], n0, kw["m0"], nb)
    assert relerr(h, hr) < 1e-12
    # the final state represents the raw one: exp(m) n' is the raw scalar normaliser
    f = np.exp(oracle.log_sigmoid(kw["fgate"]))
    i = np.exp(kw["igate"])
    nr = np.exp(kw["m0"]) * n0
    for t in range(q.shape[2]):
        nr = f[:, :, t] * nr + i[:, :, t]
    assert relerr(np.exp(m) * n, nr) < 1e-12


def test_scalar_normaliser_closed_form_of_n():
    # n_t (raw) = sum_{s<=t} exp(b_t - b_s + itilde_s) + exp(b_t) n_0, b = cumulative log f
    rng = np.random.default_rng(22)
    q, k, v, kw = rand_case(rng, 1, 1, 12, 3, 2, 1)
    bias = np.array([0.0])
    _, _, n, m = oracle.sequential_scalar_normaliser(q, k, v, kw["igate"], kw["fgate"], bias)
    lf = oracle.log_sigmoid(kw["fgate"][0, 0])
    bc = np.cumsum(lf)
    raw = np.sum(np.exp(bc[-1] - bc + kw["igate"][0, 0]))
    assert abs(math.exp(m[0, 0]) * n[0, 0] - raw) / raw < 1e-12


@pytest.mark.parametrize("bias", [0.0, 2.5, -7.0])
def test_scalar_normaliser_hand_example(bias):
    # f = 1 (ftilde = 40), itilde = 0, q = k = v = 1, dk = dv = 1: C_t = n_t = t,
    # h_t = t / max(|t + bias|, 1)
    S = 9
    ones = np.ones((1, 1, S, 1))
    h, C, n, m = oracle.sequential_scalar_normaliser(ones, ones, ones, np.zeros((1, 1, S)),
                                                     np.full((1, 1, S), 40.0), np.array([bias]))
    t = np.arange(1, S + 1)
    assert np.max(np.abs(h[0, 0, :, 0] - t / np.maximum(np.abs(t + bias), 1.0))) < 1e-12
