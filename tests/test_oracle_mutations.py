"""Each plausible mistake, planted in the oracle on the CPU, must fail a pin.

The mutations are applied with monkeypatch to a copy of one oracle function;
the pin that should catch it is run and must raise.  A mistake inside a
longer function is planted by editing one line of that function's own source
and compiling the result in the oracle's namespace.
"""

import inspect
import math
import textwrap

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


def _source_mutant(name, old, new):
    """The oracle function ``name`` with its one occurrence of ``old``
    replaced by ``new``, compiled against the oracle module's globals."""
    src = textwrap.dedent(inspect.getsource(getattr(O, name)))
    assert src.count(old) == 1, (name, old)
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant of {name}>", "exec"), ns)
    return ns[name]


SOURCE_CASES = [
    # the short last chunk of a ragged length is dropped
    ("attend_round", "n_c = -(-L // c)", "n_c = L // c",
     lambda: P.test_brute_force_small(20, 8, 4, 2, True)),
    # causal mask pointing the wrong way (a key in the past is hidden)
    ("attend_round", "np.where(kp > qp, -np.inf, s)", "np.where(kp < qp, -np.inf, s)",
     lambda: P.test_brute_force_small(16, 4, 4, 2, True)),
    # the bucket-equality mask is never applied
    ("attend_round", "if bucket_r is not None:", "if False:", P.test_bucket_mask_brute_force),
    # the duplicate count ignores the look-back chunk
    ("duplicate_counts", "(diff == 0) | (diff == 1)", "(diff == 0)", P.test_dedup_gives_set_union),
    # the routing-style assignment takes |x . mu| like the rotation hash
    ("kmeans_head", "np.argmax(p, axis=1)", "np.argmax(np.abs(p), axis=1)",
     P.test_kmeans_with_plus_minus_rotation_is_the_lsh_hash),
    # ... or the smallest dot product
    ("kmeans_head", "np.argmax(p, axis=1)", "np.argmin(p, axis=1)",
     P.test_kmeans_picks_the_largest_coordinate_with_basis_centroids),
    # the margin is taken against the smallest entry, not the runner-up
    ("hash_head", "top2[:, 1] - top2[:, 0]", "top2[:, 1] - z.min(axis=1)", P.test_hash_golden_tiny),
    # no gradient through the key normalisation
    ("backward_head", "X / torch.where(norm > 0, norm, 1.0)[:, None]",
     "X.detach() / torch.where(norm > 0, norm, 1.0).detach()[:, None]",
     lambda: P.test_backward_matches_finite_differences(False)),
    # the causal mask left out of the backward's forward
    ("backward_head", "if causal:", "if False:",
     lambda: P.test_backward_matches_finite_differences(True)),
    # combine weights normalised over positions instead of rounds
    ("backward_head", "torch.softmax(Lr, dim=0)", "torch.softmax(Lr, dim=1)",
     P.test_backward_of_v_is_the_attention_transpose),
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant may divide by zero
@pytest.mark.parametrize("name,old,new,pin", SOURCE_CASES,
                         ids=[f"{c[0]}-{i}" for i, c in enumerate(SOURCE_CASES)])
def test_pin_catches_source_mutation(monkeypatch, name, old, new, pin):
    monkeypatch.setattr(O, name, _source_mutant(name, old, new))
    with pytest.raises(AssertionError):
        pin()


def test_source_mutant_without_change_passes(monkeypatch):
    # The mutation harness itself leaves a function intact when nothing is
    # replaced: the recompiled copy must still satisfy its pins.
    monkeypatch.setattr(O, "attend_round", _source_mutant("attend_round", "n_c = -(-L // c)",
                                                          "n_c = -(-L // c)"))
    P.test_brute_force_small(20, 8, 4, 2, True)
    P.test_bucket_mask_brute_force()
