"""Each plausible mistake, planted in the oracle on the CPU, must fail a pin.

The mutations are applied with monkeypatch to a copy of one oracle function;
the pin that should catch it is run and must raise.
"""

import math

import numpy as np
import pytest

from oracle import lsh_oracle as O

import test_oracle_pins as P


def _no_lookback(k, chunk_len, L):
    return k * chunk_len, min((k + 1) * chunk_len, L)


def _wrap_lookback(k, chunk_len, L):
    return (k - 1) * chunk_len if k > 0 else 0, \
        min((k + 1) * chunk_len + (chunk_len if k == 0 else 0), L)


def _unnormalised_keys(x):
    return x


def _unstable_sort(buckets):
    n_h, L = buckets.shape
    perm = np.empty((n_h, L), np.int64)
    undo = np.empty((n_h, L), np.int64)
    for r in range(n_h):
        perm[r] = np.lexsort((-np.arange(L), buckets[r]))  # positions reversed in a bucket
        undo[r, perm[r]] = np.arange(L)
    return perm, undo


def _mean_combine(o_rounds, lse_rounds):
    m = np.max(lse_rounds, axis=0)
    lse = m + np.log(np.sum(np.exp(lse_rounds - m), axis=0))
    return o_rounds.mean(axis=0), lse


def _hash_without_negation(x, rotations, n_buckets):
    L = x.shape[0]
    n_h = rotations.shape[0]
    b = np.empty((n_h, L), np.int64)
    m = np.zeros((n_h, L))
    for r in range(n_h):
        p = x @ rotations[r]
        b[r] = np.argmax(np.concatenate([p, p], axis=1), axis=1)
    return b, m


CASES = [
    ("window_slots", _no_lookback, lambda: P.test_brute_force_small(16, 4, 4, 2, True)),
    ("window_slots", _wrap_lookback, lambda: P.test_brute_force_small(24, 8, 6, 3, False)),
    ("normalised_keys", _unnormalised_keys, P.test_attention_golden_tiny),
    ("sort_head", _unstable_sort, P.test_sort_matches_tuple_sort_and_invariants),
    ("combine_head", _mean_combine, lambda: P.test_multiset_union_closed_form(False)),
    ("hash_head", _hash_without_negation, P.test_hash_golden_tiny),
]


@pytest.mark.parametrize("name,mutant,pin", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_pin_catches_mutation(monkeypatch, name, mutant, pin):
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()


def test_pin_catches_missing_scale(monkeypatch):
    real = O.attend_round

    def no_scale(x, v, perm_r, chunk_len, causal, dedup_undo=None, bucket_r=None):
        return real(x * math.sqrt(x.shape[1]), v, perm_r, chunk_len, causal, dedup_undo,
                    bucket_r)

    monkeypatch.setattr(O, "attend_round", no_scale)
    with pytest.raises(AssertionError):
        P.test_attention_golden_tiny()


def test_pin_catches_wrong_self_constant(monkeypatch):
    monkeypatch.setattr(O, "SELF_SCORE", -1e5 + 0.5)
    with pytest.raises(AssertionError):
        P.test_attention_golden_tiny()
