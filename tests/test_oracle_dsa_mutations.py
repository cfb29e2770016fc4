"""Planted mistakes in the DSA oracle: each test swaps one plausible error into
oracle/dsa_oracle.py (on the CPU, through monkeypatch) and checks that at least one
pin in test_oracle_dsa.py catches it, so the pins constrain every step of the
indexer, the token top-k and the attention over the chosen tokens."""
import math

import pytest
import torch

import oracle
import oracle.dsa_oracle as D
from tests import test_oracle_dsa as pins


@pytest.fixture
def patch(monkeypatch):
    """Set a name in the DSA oracle module and in the package that re-exports it."""
    def setattr_both(name, value):
        monkeypatch.setattr(D, name, value)
        if hasattr(oracle, name):
            monkeypatch.setattr(oracle, name, value)
    return setattr_both


def _caught(*tests):
    for t in tests:
        try:
            t()
        except AssertionError:
            return True
    return False


ALL = (pins.test_indexer_closed_form, pins.test_indexer_heads_add_with_their_weights,
       pins.test_select_tokens_matches_a_full_sort_with_ties, pins.test_all_tokens_selected_is_full_causal_attention,
       pins.test_selection_and_future_tokens)


def test_pins_pass_on_the_unmodified_oracle():
    assert not _caught(*ALL)


def test_indexer_without_relu_is_caught(patch):
    patch("indexer_scores", lambda q_i, k_i, w_i, t: (k_i[: t + 1].double() @ q_i.double().T) @ w_i.double())
    assert _caught(*ALL)


def test_indexer_without_head_weights_is_caught(patch):
    patch("indexer_scores", lambda q_i, k_i, w_i, t: torch.relu(k_i[: t + 1].double() @ q_i.double().T).sum(1))
    assert _caught(*ALL)


def test_indexer_reading_one_future_key_is_caught(patch):
    real = D.indexer_scores
    patch("indexer_scores", lambda q_i, k_i, w_i, t: real(q_i, k_i, w_i, min(t + 1, k_i.shape[0] - 1)))
    assert _caught(*ALL)


def test_ties_to_the_higher_index_are_caught(patch):
    def bad(score, k):
        n = score.shape[0]
        if n <= k:
            return list(range(n))
        return sorted(sorted(range(n), key=lambda s: (-float(score[s]), -s))[:k])
    patch("select_tokens", bad)
    assert _caught(*ALL)


def test_lowest_scores_kept_is_caught(patch):
    def bad(score, k):
        n = score.shape[0]
        if n <= k:
            return list(range(n))
        return sorted(sorted(range(n), key=lambda s: (float(score[s]), s))[:k])
    patch("select_tokens", bad)
    assert _caught(*ALL)


def test_one_token_short_is_caught(patch):
    real = D.select_tokens
    patch("select_tokens", lambda score, k: real(score, k)[:-1] if score.shape[0] > 1 else real(score, k))
    assert _caught(*ALL)


def test_missing_softmax_scale_is_caught(patch):
    real = D.attend
    patch("attend", lambda qh, K, V, scale: real(qh, K, V, 1.0))
    assert _caught(*ALL)


def test_scale_of_the_value_dim_is_caught(patch):
    real = D.attend
    patch("attend", lambda qh, K, V, scale: real(qh, K, V, 1.0 / math.sqrt(V.shape[1])))
    assert _caught(*ALL)
