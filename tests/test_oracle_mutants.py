"""The oracle's pins catch plausible mistakes.

Each test plants one mistake in the oracle (on the CPU, through monkeypatch,
undone when the test ends) and checks that a pin of tests/test_oracle.py or
tests/test_oracle_dropout.py fails on it: a dropped scale, an off-by-one in
the causal mask, a missing -D term, dV without the transpose, the dropout
factor forgotten, the keep-mask words and bytes swapped, a Philox round too
few, an off-by-one in the key-padding length, and a bias added before the
scale.
"""
import numpy as np
import pytest

import oracle
import oracle.attention as att
from oracle import philox
from tests import test_oracle as pins
from tests import test_oracle_dropout as dpins

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_pins_pass_on_the_unmodified_oracle():
    pins.test_forward_matches_torch_sdpa(2, 3, 33, 16, True)
    pins.test_backward_matches_finite_differences(5, 4, True)
    pins.test_key_padding_matches_torch_autograd(True)
    dpins.test_keep_mask_layout_per_element()
    dpins.test_dropout_backward_matches_torch_autograd(True)
    dpins.test_philox_known_answers()


def test_dropped_scale_is_caught(monkeypatch):
    orig = att.head_probs
    monkeypatch.setattr(att, "head_probs", lambda q, k, scale, *a, **kw: orig(q, k, 1.0, *a, **kw))
    _fails(pins.test_forward_matches_torch_sdpa, 2, 3, 33, 16, True)


def test_causal_off_by_one_is_caught(monkeypatch):
    def strict(nq, nk, rows=None):
        rows = np.arange(nq) if rows is None else np.asarray(rows)
        return np.arange(nk)[None, :] < (rows[:, None] + (nk - nq))  # should be <=
    monkeypatch.setattr(att, "causal_visible", strict)
    _fails(pins.test_forward_matches_torch_sdpa, 2, 3, 33, 16, True)


def _backward_with(mistake):
    """head_backward restated with one planted mistake."""
    def hb(q, k, v, do, scale, causal, keep_fn=None, kscale=1.0, nk_valid=None, bias=None):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
        p, _ = att.head_probs(q, k, scale, causal, None, None, nk_valid)
        o = p @ v
        D = (do * o).sum(axis=1)
        dp = do @ v.T
        ds = p * dp if mistake == "no_D" else p * (dp - D[:, None])
        dv = (p @ do[: p.shape[1]] if p.shape[0] == p.shape[1] else p.T @ do) \
            if mistake == "no_transpose" else p.T @ do
        return scale * ds @ k, scale * ds.T @ q, dv, D
    return hb


@pytest.mark.parametrize("mistake", ["no_D", "no_transpose"])
def test_backward_mistakes_are_caught(monkeypatch, mistake):
    hb = _backward_with(mistake)
    monkeypatch.setattr(att, "head_backward", hb)
    monkeypatch.setattr(oracle, "head_backward", hb)
    _fails(pins.test_backward_matches_finite_differences, 5, 4, True)


def test_forgotten_dropout_factor_is_caught(monkeypatch):
    monkeypatch.setattr(philox, "keep_scale", lambda p: 1.0)
    _fails(dpins.test_dropout_backward_matches_torch_autograd, True)
    _fails(dpins.test_dropout_is_unbiased_on_average)


def test_swapped_keep_mask_layout_is_caught(monkeypatch):
    orig = philox.keep_mask
    # rows and columns exchanged when picking the word and the byte
    monkeypatch.setattr(philox, "keep_mask", lambda bh, r, c, p, s, o: orig(bh, c, r, p, s, o).T)
    _fails(dpins.test_keep_mask_layout_per_element)


def test_missing_philox_round_is_caught(monkeypatch):
    orig = philox.philox4x32_10

    def nine_rounds(ctr, key):
        # the published rounds, one fewer
        ctr = np.asarray(ctr, dtype=np.uint64) & philox._MASK32
        key = np.asarray(key, dtype=np.uint64) & philox._MASK32
        c0, c1, c2, c3 = (ctr[..., n].copy() for n in range(4))
        k0, k1 = key[..., 0].copy(), key[..., 1].copy()
        for rnd in range(9):
            if rnd > 0:
                k0 = (k0 + philox.W0) & philox._MASK32
                k1 = (k1 + philox.W1) & philox._MASK32
            p0 = c0 * np.uint64(philox.M0)
            p1 = c2 * np.uint64(philox.M1)
            c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & philox._MASK32,
                              (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & philox._MASK32)
        return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)

    assert orig is not nine_rounds
    monkeypatch.setattr(philox, "philox4x32_10", nine_rounds)
    _fails(dpins.test_philox_known_answers)


def test_key_padding_off_by_one_is_caught(monkeypatch):
    orig = att.head_probs

    def plus_one(q, k, scale, causal, rows=None, nq_total=None, nk_valid=None, bias=None):
        return orig(q, k, scale, causal, rows, nq_total, None if nk_valid is None else nk_valid + 1,
                    bias)
    monkeypatch.setattr(att, "head_probs", plus_one)
    _fails(pins.test_key_padding_matches_torch_autograd, True)


def test_bias_before_scale_is_caught(monkeypatch):
    """The bias belongs to the scaled scores; adding it before the scale (so
    that it gets scaled too) must fail the SDPA pin."""
    orig = att.head_probs

    def scaled_bias(q, k, scale, causal, rows=None, nq_total=None, nk_valid=None, bias=None):
        return orig(q, k, scale, causal, rows, nq_total, nk_valid,
                    None if bias is None else np.asarray(bias) * scale)
    monkeypatch.setattr(att, "head_probs", scaled_bias)
    _fails(pins.test_bias_matches_torch_autograd, False)
