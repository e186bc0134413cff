"""Planted mistakes in copies of the NEXT-row oracles: each copy must fail at least one pin.

GDN-2: a copy of the token-by-token recurrence with one switch per mistake, run through every
pin of tests/test_oracle_gdn2.py.  Rotation Theta and GroupNorm + gate: mistaken copies put in
place of the oracle's functions while the pins of tests/test_oracle_retention_block.py run."""
import numpy as np
import pytest

import oracle
from tests import test_oracle_gdn2 as gdn2_pins
from tests import test_oracle_retention_block as block_pins


def gdn2_variant(mistake=None):
    def seq(q, k, v, g, b, w, S0=None):
        q, k, v, g, b, w = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, b, w))
        B, H, T, K = q.shape
        V = v.shape[-1]
        S = np.zeros((B, H, K, V)) if S0 is None else np.array(S0, dtype=np.float64)
        o = np.zeros((B, H, T, V))
        for t in range(T):
            kt, bt, qt = k[:, :, t], b[:, :, t], q[:, :, t]
            ut = v[:, :, t] if mistake == "write_gate_dropped" else w[:, :, t] * v[:, :, t]
            if mistake == "erase_gate_dropped":
                bt = np.ones_like(bt)
            dec = np.exp(g[:, :, t])[..., None]
            Sd = S if mistake == "decay_after_update" else dec * S
            src = S if mistake == "read_before_decay" else Sd
            if mistake == "erase_and_read_swapped":
                r = np.einsum("bhkv,bhk->bhv", src, bt * kt)
                erase = np.einsum("bhk,bhv->bhkv", kt, r)
            else:
                r = np.einsum("bhkv,bhk->bhv", src, kt)
                erase = np.einsum("bhk,bhv->bhkv", bt * kt, r)
            if mistake == "erase_sign":
                erase = -erase
            Snew = Sd - erase + np.einsum("bhk,bhv->bhkv", kt, ut)
            if mistake == "decay_after_update":
                Snew = dec * Snew
            read_from = Sd if mistake == "readout_before_update" else Snew
            o[:, :, t] = np.einsum("bhkv,bhk->bhv", read_from, qt)
            S = Snew
        return o, S
    return seq


GDN2_MISTAKES = ["erase_and_read_swapped", "decay_after_update", "write_gate_dropped", "erase_gate_dropped",
                 "read_before_decay", "readout_before_update", "erase_sign"]


def test_gdn2_copy_without_mistakes_is_the_oracle():
    args = gdn2_pins._inputs(11, T=25)
    o1, S1 = oracle.gdn2_sequential(*args)
    o2, S2 = gdn2_variant()(*args)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(S2, S1, atol=1e-12)
    for pin in gdn2_pins.PINS:
        pin(gdn2_variant())


def fails_a_pin(pins, *call):
    for pin in pins:
        try:
            pin(*call)
        except AssertionError:
            return pin.__name__
    return None


@pytest.mark.parametrize("mistake", GDN2_MISTAKES)
def test_gdn2_pins_catch(mistake):
    assert fails_a_pin(gdn2_pins.PINS, gdn2_variant(mistake)), mistake


# ---------------------------------------------------------------- rotation and GroupNorm
def rotate_variant(mistake):
    def rot(x, pos0=None, base=10000.0):
        x = np.asarray(x, dtype=np.float64)
        B, NH, S, D = x.shape
        pos0 = np.zeros(B, dtype=np.int64) if pos0 is None else np.asarray(pos0, dtype=np.int64)
        expo = (-1.0 if mistake == "frequency_exponent" else -2.0) * np.arange(D // 2) / D
        theta = base ** expo
        out = np.empty_like(x)
        for b in range(B):
            pos = (pos0[b] + np.arange(S) + (1 if mistake == "position_from_one" else 0)).astype(np.float64)
            ang = pos[:, None] * theta[None, :]
            c, s = np.cos(ang), np.sin(ang)
            if mistake == "opposite_sense":
                s = -s
            if mistake == "halves_not_pairs":
                i0, i1 = slice(0, D // 2), slice(D // 2, D)
            else:
                i0, i1 = slice(0, D, 2), slice(1, D, 2)
            x0, x1 = x[b, :, :, i0], x[b, :, :, i1]
            out[b, :, :, i0] = x0 * c - x1 * s
            out[b, :, :, i1] = x0 * s + x1 * c
        return out
    return rot


def gn_variant(mistake):
    def gn(h, g=None, weight=None, bias=None, eps=1e-5):
        h = np.asarray(h, dtype=np.float64)
        B, NH, S, DHV = h.shape
        axis = 2 if mistake == "over_tokens" else -1
        mu = h.mean(axis=axis, keepdims=True)
        var = h.var(axis=axis, keepdims=True, ddof=1 if mistake == "unbiased_variance" else 0)
        y = (h - mu) / (np.sqrt(var) + eps if mistake == "eps_outside_sqrt" else np.sqrt(var + eps))
        if weight is not None:
            y = y * np.asarray(weight, dtype=np.float64).reshape(1, NH, 1, DHV)
        if bias is not None:
            y = y + np.asarray(bias, dtype=np.float64).reshape(1, NH, 1, DHV)
        if g is not None:
            gg = np.asarray(g, dtype=np.float64)
            y = y * (1 / (1 + np.exp(-gg)) if mistake == "sigmoid_gate" else oracle.silu(gg))
        return y
    return gn


BLOCK_PINS = [block_pins.test_rotation_is_complex_multiplication,
              block_pins.test_rotation_position_zero_is_identity_and_norms_are_kept,
              block_pins.test_rotated_scores_depend_on_relative_position_only,
              block_pins.test_group_norm_gate_matches_torch, block_pins.test_group_norm_invariants,
              block_pins.test_retention_block_is_shift_invariant,
              block_pins.test_retention_block_composes_the_pinned_steps,
              lambda: block_pins.test_rotation_first_pair_turns_by_the_position(64)]


@pytest.mark.parametrize("mistake", ["frequency_exponent", "position_from_one", "opposite_sense", "halves_not_pairs"])
def test_rotation_pins_catch(mistake, monkeypatch):
    monkeypatch.setattr(oracle, "theta_rotate", rotate_variant(mistake))
    assert fails_a_pin(BLOCK_PINS), mistake


@pytest.mark.parametrize("mistake", ["over_tokens", "unbiased_variance", "eps_outside_sqrt", "sigmoid_gate"])
def test_group_norm_pins_catch(mistake, monkeypatch):
    monkeypatch.setattr(oracle, "group_norm_gate", gn_variant(mistake))
    assert fails_a_pin(BLOCK_PINS), mistake


def test_unmutated_copies_pass_the_block_pins(monkeypatch):
    monkeypatch.setattr(oracle, "theta_rotate", rotate_variant(None))
    monkeypatch.setattr(oracle, "group_norm_gate", gn_variant(None))
    assert fails_a_pin(BLOCK_PINS) is None
