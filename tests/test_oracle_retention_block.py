"""Pins for the steps either side of retention in the oracle (Edifice.Attention.RetNet, "Key
Innovation" and "Multi-Scale Retention (MSR)"): the rotation Theta of q and k, the per-head
GroupNorm, the SiLU gate and their composition with the recurrence.  Each pin ties the
oracle to something other than its own formula: complex arithmetic, torch's GroupNorm and
SiLU, exact invariants of a rotation and of retention."""
import numpy as np
import pytest
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def test_rotation_is_complex_multiplication():
    """Entries (2j, 2j+1) as one complex number times e^{i p theta_j}, theta_j a geometric
    sequence from 1 down to base^{-(D-2)/D}, computed by numpy's complex exponential."""
    rng = _rng(1)
    B, NH, S, D = 2, 3, 17, 12
    x = rng.standard_normal((B, NH, S, D))
    pos0 = np.array([0, 1000])
    base = 500.0
    got = oracle.theta_rotate(x, pos0, base)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    freq = np.geomspace(1.0, base ** (-(D - 2) / D), D // 2)
    for b in range(B):
        p = pos0[b] + np.arange(S)
        zr = z[b] * np.exp(1j * np.outer(p, freq))[None]
        np.testing.assert_allclose(got[b, ..., 0::2], zr.real, rtol=0, atol=1e-11)
        np.testing.assert_allclose(got[b, ..., 1::2], zr.imag, rtol=0, atol=1e-11)


def test_rotation_position_zero_is_identity_and_norms_are_kept():
    rng = _rng(2)
    x = rng.standard_normal((1, 2, 1, 16))
    np.testing.assert_array_equal(oracle.theta_rotate(x), x)
    y = rng.standard_normal((1, 2, 40, 16))
    r = oracle.theta_rotate(y, np.array([123]))
    np.testing.assert_allclose(r[..., 0::2] ** 2 + r[..., 1::2] ** 2, y[..., 0::2] ** 2 + y[..., 1::2] ** 2,
                               rtol=1e-12)


def test_rotated_scores_depend_on_relative_position_only():
    """(Q Theta)(K Theta)^T is unchanged when every position moves by the same amount; a
    rotation of k in the opposite sense would make it depend on n + m instead."""
    rng = _rng(3)
    q = rng.standard_normal((1, 1, 24, 8))
    k = rng.standard_normal((1, 1, 24, 8))
    s0 = oracle.theta_rotate(q, np.array([0]))[0, 0] @ oracle.theta_rotate(k, np.array([0]))[0, 0].T
    s1 = oracle.theta_rotate(q, np.array([777]))[0, 0] @ oracle.theta_rotate(k, np.array([777]))[0, 0].T
    np.testing.assert_allclose(s1, s0, rtol=1e-9, atol=1e-9)
    # the diagonal is the unrotated q . k
    np.testing.assert_allclose(np.diag(s0), np.einsum("sd,sd->s", q[0, 0], k[0, 0]), rtol=1e-12, atol=1e-12)


def test_group_norm_gate_matches_torch():
    """Each head of each token is one group of DHV channels: torch.nn.functional.group_norm
    with NH groups over NH*DHV channels per (batch, token), then torch's SiLU."""
    rng = _rng(4)
    B, NH, S, DHV = 2, 3, 5, 8
    h = rng.standard_normal((B, NH, S, DHV)) * 3 + 1
    g = rng.standard_normal((B, NH, S, DHV))
    w = rng.standard_normal(NH * DHV)
    bb = rng.standard_normal(NH * DHV)
    eps = 1e-3
    got = oracle.group_norm_gate(h, g, w, bb, eps)
    x = torch.from_numpy(h).permute(0, 2, 1, 3).reshape(B * S, NH * DHV)
    ref = torch.nn.functional.group_norm(x, NH, torch.from_numpy(w), torch.from_numpy(bb), eps)
    ref = ref.reshape(B, S, NH, DHV).permute(0, 2, 1, 3)
    ref = ref * torch.nn.functional.silu(torch.from_numpy(g))
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_group_norm_invariants():
    rng = _rng(5)
    h = rng.standard_normal((1, 2, 7, 16))
    eps = 1e-2
    y = oracle.group_norm_gate(h, eps=eps)
    np.testing.assert_allclose(y.mean(axis=-1), 0, atol=1e-13)
    var = h.var(axis=-1)
    np.testing.assert_allclose(y.var(axis=-1), var / (var + eps), rtol=1e-12)
    # shift invariance of each group, and a gate of 0 gives 0
    np.testing.assert_allclose(oracle.group_norm_gate(h + 5.0, eps=eps), y, atol=1e-12)
    assert np.all(oracle.group_norm_gate(h, np.zeros_like(h), eps=eps) == 0)
    # silu(x) - silu(-x) = x
    x = np.linspace(-20, 20, 101)
    np.testing.assert_allclose(oracle.silu(x) - oracle.silu(-x), x, atol=1e-12)


def test_retention_block_is_shift_invariant():
    """With a zero initial state, retention of rotated q, k depends on positions only through
    differences, so moving pos0 leaves the block's output unchanged."""
    rng = _rng(6)
    B, NH, S, D = 2, 2, 20, 8
    q, k, v = (rng.standard_normal((B, NH, S, D)) for _ in range(3))
    g = rng.standard_normal((B, NH, S, D))
    y0, C0_, _, _ = oracle.retention_block(q, k, v, g=g, pos0=np.array([0, 0]))
    y1, C1_, _, _ = oracle.retention_block(q, k, v, g=g, pos0=np.array([50, 9000]))
    np.testing.assert_allclose(y1, y0, rtol=1e-8, atol=1e-8)


def test_retention_block_composes_the_pinned_steps():
    """Rotation -> recurrence -> GroupNorm -> gate, checked against the brute-force parallel
    form (pinned separately) on the rotated inputs, in mLSTM mode too."""
    rng = _rng(7)
    B, NH, S, D = 1, 2, 16, 8
    q, k, v = (rng.standard_normal((B, NH, S, D)) for _ in range(3))
    ig, fg = rng.standard_normal((B, NH, S)), rng.standard_normal((B, NH, S)) + 2
    g = rng.standard_normal((B, NH, S, D))
    for retention in (True, False):
        y, _, _, _ = oracle.retention_block(q, k, v, ig, fg, g=g, pos0=np.array([3]), retention=retention,
                                            eps=1e-4)
        qr, kr = oracle.theta_rotate(q, np.array([3])), oracle.theta_rotate(k, np.array([3]))
        h = oracle.parallel_form(qr, kr, v, None if retention else ig, None if retention else fg,
                                 retention=retention)[0]
        np.testing.assert_allclose(y, oracle.group_norm_gate(h, g, eps=1e-4), rtol=1e-7, atol=1e-7)


@pytest.mark.parametrize("D", [2, 64])
def test_rotation_first_pair_turns_by_the_position(D):
    """theta_0 = 1: the first pair of a unit vector (1, 0) at position p is (cos p, sin p)."""
    x = np.zeros((1, 1, 1, D))
    x[..., 0] = 1
    r = oracle.theta_rotate(x, np.array([5]))
    assert abs(r[0, 0, 0, 0] - np.cos(5.0)) < 1e-15 and abs(r[0, 0, 0, 1] - np.sin(5.0)) < 1e-15
