"""Pins for the Gated DeltaNet-2 oracle (burn-gdn2 config.rs): the roles the page gives the two
gates (b: how much of each key channel to erase; w: how much of each value channel to write),
the reductions it states (b = w = beta 1 is KDA, whose delta rule stores v under k exactly at
beta = 1; a scalar decay gives Gated DeltaNet), associative recall, a hand-worked example and
the chunked evaluation against the token-by-token one."""
import numpy as np
import pytest

import oracle


def _inputs(seed, B=1, H=2, T=40, K=8, V=6, decay=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, K))
    k = rng.standard_normal((B, H, T, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, V))
    g = -np.abs(rng.standard_normal((B, H, T, K))) * decay
    b = 1 / (1 + np.exp(-rng.standard_normal((B, H, T, K))))
    w = 1 / (1 + np.exp(-rng.standard_normal((B, H, T, V))))
    S0 = rng.standard_normal((B, H, K, V))
    return q, k, v, g, b, w, S0


def pin_hand_example(seq):
    """K = V = 1, q = k = v = 1, alpha = 1/2, b = 1/2, w = 1, S0 = 0:
    S_1 = 1, S_2 = 1/2 - 1/4 + 1 = 1.25, S_3 = 0.625 - 0.3125 + 1 = 1.3125 (-> 4/3)."""
    T = 3
    ones = np.ones((1, 1, T, 1))
    o, S = seq(ones, ones, ones, np.log(0.5) * ones, 0.5 * ones, ones)
    np.testing.assert_allclose(o[0, 0, :, 0], [1.0, 1.25, 1.3125], rtol=0, atol=1e-15)
    assert abs(S[0, 0, 0, 0] - 1.3125) < 1e-15


def pin_associative_recall_with_one_hot_keys(seq):
    """No decay, full erase and write, one-hot keys: the state is a key -> value table; writing
    a key again replaces its value (the delta rule's overwrite) and other keys keep theirs."""
    K, V = 5, 3
    keys = [0, 3, 1, 3, 4]
    rng = np.random.default_rng(1)
    vals = rng.standard_normal((len(keys), V))
    T = len(keys)
    k = np.zeros((1, 1, T, K))
    for t, i in enumerate(keys):
        k[0, 0, t, i] = 1
    ones_k, ones_v = np.ones((1, 1, T, K)), np.ones((1, 1, T, V))
    _, S = seq(k, k, vals[None, None], 0 * ones_k, ones_k, ones_v)
    latest = {i: vals[t] for t, i in enumerate(keys)}
    for i in range(K):
        np.testing.assert_allclose(S[0, 0, i], latest.get(i, np.zeros(V)), atol=1e-15)


def pin_kda_reduction_stores_v_under_k(seq):
    """b = w = 1 (KDA with beta = 1) and a unit key: right after the step the memory returns
    exactly v for k, whatever it held before (the delta rule's error-correcting write)."""
    q, k, v, g, b, w, S0 = _inputs(2, T=1)
    _, S = seq(q, k, v, g, np.ones_like(b), np.ones_like(w), S0)
    got = np.einsum("bhkv,bhk->bhv", S, k[:, :, 0])
    np.testing.assert_allclose(got, v[:, :, 0], atol=1e-13)


def pin_erase_gate_acts_per_key_channel(seq):
    """No write (w = 0), no decay: a key channel with b_i = 0 keeps its row of the state; with
    the erase applied, k^T S drops by the factor 1 - sum_i b_i k_i^2."""
    q, k, v, g, b, w, S0 = _inputs(3, T=1)
    b[..., 2] = 0.0
    _, S = seq(q, k, v, 0 * g, b, 0 * w, S0)
    np.testing.assert_array_equal(S[..., 2, :], S0[..., 2, :])
    kk = k[:, :, 0]
    before = np.einsum("bhkv,bhk->bhv", S0, kk)
    after = np.einsum("bhkv,bhk->bhv", S, kk)
    factor = 1 - np.sum(b[:, :, 0] * kk * kk, axis=-1)
    np.testing.assert_allclose(after, factor[..., None] * before, atol=1e-13)


def pin_write_gate_acts_per_value_channel(seq):
    """From a zero state, value channel j of the state and of o is linear in w_j: w_j = 0 leaves
    it zero and halving w_j halves it, the other channels unchanged."""
    q, k, v, g, b, w, _ = _inputs(4)
    o1, S1 = seq(q, k, v, g, b, w)
    w2 = w.copy()
    w2[..., 1] *= 0.5
    w2[..., 4] = 0.0
    o2, S2 = seq(q, k, v, g, b, w2)
    np.testing.assert_allclose(o2[..., 1], 0.5 * o1[..., 1], atol=1e-12)
    assert np.all(o2[..., 4] == 0) and np.all(S2[..., 4] == 0)
    np.testing.assert_allclose(o2[..., [0, 2, 3, 5]], o1[..., [0, 2, 3, 5]], atol=1e-12)


def pin_channel_decay_and_the_scalar_case(seq):
    """With nothing erased or written, each key row of the state decays by its own channel's
    product of alpha; a scalar decay (Gated DeltaNet) scales the whole state."""
    q, k, v, g, b, w, S0 = _inputs(5)
    _, S = seq(q, k, v, g, 0 * b, 0 * w, S0)
    np.testing.assert_allclose(S, np.exp(g.sum(axis=2))[..., None] * S0, rtol=1e-12)
    gs = np.repeat(g[..., :1], g.shape[-1], axis=-1)
    _, S = seq(q, k, v, gs, 0 * b, 0 * w, S0)
    np.testing.assert_allclose(S, np.exp(gs[..., 0].sum(axis=2))[..., None, None] * S0, rtol=1e-12)


@pytest.mark.parametrize("chunk,T,decay", [(1, 20, 0.5), (4, 33, 0.5), (16, 70, 3.0), (64, 100, 0.5),
                                           (64, 130, 20.0)])
def test_chunked_equals_sequential(chunk, T, decay):
    """The chunked evaluation (triangular solve per chunk) equals the recurrence, ragged last
    chunk and strong decays (log alpha down to about -60 per token) included."""
    args = _inputs(6, T=T, decay=decay)
    o1, S1 = oracle.gdn2_sequential(*args)
    o2, S2 = oracle.gdn2_chunk(*args, chunk=chunk)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-10)


def pin_split_and_resume_and_linearity(seq):
    q, k, v, g, b, w, S0 = _inputs(7, T=30)
    o, S = seq(q, k, v, g, b, w, S0)
    sl1, sl2 = (slice(None), slice(None), slice(0, 12)), (slice(None), slice(None), slice(12, None))
    oa, Sa = seq(q[sl1], k[sl1], v[sl1], g[sl1], b[sl1], w[sl1], S0)
    ob, Sb = seq(q[sl2], k[sl2], v[sl2], g[sl2], b[sl2], w[sl2], Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=2), o, atol=1e-12)
    np.testing.assert_allclose(Sb, S, atol=1e-12)
    o3, S3 = seq(q, k, 3 * v, g, b, w, 3 * S0)
    np.testing.assert_allclose(o3, 3 * o, atol=1e-11)


# Each pin above, on the oracle.  tests/test_oracle_mutations_next.py runs the same pins on
# copies of the recurrence with planted mistakes and expects every copy to fail one of them.
PINS = [pin_hand_example, pin_associative_recall_with_one_hot_keys, pin_kda_reduction_stores_v_under_k,
        pin_erase_gate_acts_per_key_channel, pin_write_gate_acts_per_value_channel,
        pin_channel_decay_and_the_scalar_case, pin_split_and_resume_and_linearity]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.gdn2_sequential)
