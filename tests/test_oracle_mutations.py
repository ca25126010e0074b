"""Planted mistakes in the oracle (on the CPU) must be caught by its pins.

Each case swaps one oracle function for a plausible wrong variant -- a flipped
sign, a dropped term, a wrong composition order, a wrong pooling -- and checks that
at least one pin test then fails.  This shows the pins constrain the oracle beyond
re-stating it.
"""
import numpy as np
import pytest

from oracle import hla_oracle as ho
from oracle import routing_recipe as rr
import tests.test_oracle_hla as th
import tests.test_oracle_routing as tr


def _wrong_sign_step(S, k, v, alpha, beta):
    Sk = S @ k
    return alpha * (S + beta * np.outer(Sk, k)) + beta * np.outer(v, k)


def _dropped_decay_step(S, k, v, alpha, beta):
    Sk = S @ k
    return (S - beta * np.outer(Sk, k)) + beta * np.outer(v, k)


def _transposed_write_step(S, k, v, alpha, beta):
    Sk = S @ k
    return alpha * (S - beta * np.outer(Sk, k)) + beta * np.outer(k, v)


def _descending_compose(trans, gates_row, active):
    dv, dk = trans[0][1].shape
    S = np.zeros((dv, dk))
    for j in sorted(active, reverse=True):
        A, B = trans[j]
        g = float(gates_row[j])
        S = S + g * ((S @ A + B) - S)
    return S


def _ungated_b_compose(trans, gates_row, active):
    dv, dk = trans[0][1].shape
    S = np.zeros((dv, dk))
    for j in active:
        A, B = trans[j]
        g = float(gates_row[j])
        S = S + g * (S @ A - S) + B
    return S


def _mean_pool(x, tau, n_tokens=None):
    x = np.asarray(x, np.float32)
    n = x.shape[-2] if n_tokens is None else n_tokens
    return x[..., :n, :].mean(-2).astype(np.float32)


def _bad_exp(x):
    x = np.asarray(x, np.float32)
    return (np.exp(x.astype(np.float64)) * (1 + 3e-7)).astype(np.float32)


def _window_gate_mean(rq, rkw, d, bias):
    # a log-MEAN-exp over the windows instead of the log-sum-exp (drops log W)
    rkw = np.asarray(rkw, np.float32)
    t = (rr.dot32(np.asarray(rq, np.float32)[..., None, :], rkw) * rr.gate_scale(d)).astype(np.float32)
    m = t.max(axis=-1)
    s = np.zeros_like(m)
    for u in range(t.shape[-1]):
        s = (s + rr.exp32((t[..., u] - m).astype(np.float32))).astype(np.float32)
    z = ((m + rr.log32(s / np.float32(t.shape[-1]))).astype(np.float32) + np.float32(bias)).astype(np.float32)
    return (np.float32(1.0) / (np.float32(1.0) + rr.exp32(-z))).astype(np.float32)


def _window_gate_max(rq, rkw, d, bias):
    # the best window alone instead of the log-sum-exp
    rkw = np.asarray(rkw, np.float32)
    t = (rr.dot32(np.asarray(rq, np.float32)[..., None, :], rkw) * rr.gate_scale(d)).astype(np.float32)
    z = (t.max(axis=-1) + np.float32(bias)).astype(np.float32)
    return (np.float32(1.0) / (np.float32(1.0) + rr.exp32(-z))).astype(np.float32)


def _run(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


CASES = [
    ("gdn_token_step", _wrong_sign_step, ho),
    ("gdn_token_step", _dropped_decay_step, ho),
    ("gdn_token_step", _transposed_write_step, ho),
    ("compose_state", _descending_compose, ho),
    ("compose_state", _ungated_b_compose, ho),
    ("lme_pool32", _mean_pool, rr),
    ("exp32", _bad_exp, rr),
    ("gate_window32", _window_gate_mean, rr),
    ("gate_window32", _window_gate_max, rr),
]


@pytest.mark.parametrize("name,bad,mod", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, bad, mod):
    monkeypatch.setattr(mod, name, bad)
    pins = [
        (th.test_wy_form_equals_literal_transition, 16, 12, 12),
        (th.test_exact_rational_brute_force, 8, 2, 2),
        (th.test_exact_rational_brute_force, 8, 4, 3),
        (th.test_decode_matches_prefill_of_extended_sequence, 16, 0),
        (tr.test_lme_matches_float64_definition,),
        (tr.test_exp32_error_bound,),
        (tr.test_window_gate_matches_float64_definition,),
        (tr.test_window_gate_of_equal_windows_adds_log_count,),
    ]
    caught = [p[0].__name__ for p in pins if _run(*p)]
    assert caught, f"no pin caught the planted mistake in {name}"
