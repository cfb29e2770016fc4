"""Planted mistakes: each test swaps one plausible error into the CPU oracle
(on the CPU, through monkeypatch) and checks that at least one pin in
test_oracle_pins.py catches it.  This shows the pins constrain every step."""
import math

import pytest
import torch

import oracle
import oracle.nsa_oracle as O
from tests import test_oracle_pins as pins


class _Both:
    """Patch a name in the oracle module and in the package that re-exports it."""

    def __init__(self, mp):
        self.mp = mp

    def setattr(self, target, name, value):
        self.mp.setattr(target, name, value)
        if target is O and hasattr(oracle, name):
            self.mp.setattr(oracle, name, value)


@pytest.fixture
def monkeypatch(monkeypatch):  # noqa: F811 -- wraps pytest's fixture
    return _Both(monkeypatch)


def _caught(*tests):
    for t in tests:
        try:
            t()
        except AssertionError:
            return True
    return False


def test_channel_major_flattening_is_caught(monkeypatch):
    def bad_phi(X, W, l, s):
        X, W = O._f64(X), O._f64(W)
        T, d = X.shape
        n = O.num_cmp_blocks(T, l, s)
        if n == 0:
            return torch.zeros((0, W.shape[1]), dtype=O.F64)
        return torch.stack([X[s * i: s * i + l].T.reshape(l * d) for i in range(n)]) @ W
    monkeypatch.setattr(O, "phi_compress", bad_phi)
    assert _caught(pins.test_phi_matches_bruteforce_sum, pins.test_phi_selector_and_meanpool_closed_forms)


def test_visibility_off_by_one_is_caught(monkeypatch):
    def bad_vis(t, l, s, n_total):
        if t < l:
            return 0
        return min(n_total, (t - l) // s + 1)
    monkeypatch.setattr(O, "num_visible_cmp_blocks", bad_vis)
    assert _caught(pins.test_visible_blocks_match_definition, pins.test_nsa_handworked_closed_forms)


def test_single_head_scores_are_caught(monkeypatch):
    real = O.selection_scores
    monkeypatch.setattr(O, "selection_scores", lambda p, t, l, s, b, mapping="touch": real(p[:1], t, l, s, b, mapping))
    assert _caught(pins.test_nsa_handworked_closed_forms)


def test_contained_only_mapping_is_caught(monkeypatch):
    def bad(p, t, l, s, b, mapping="touch"):
        nb = t // b + 1
        score = torch.zeros(nb, dtype=O.F64)
        ph = p.sum(0)
        for i in range(ph.shape[0]):
            if (s * i) // b == (s * i + l - 1) // b:
                score[(s * i) // b] += ph[i]
        return score
    monkeypatch.setattr(O, "selection_scores", bad)
    assert _caught(pins.test_nsa_handworked_closed_forms)


def test_ties_to_higher_index_are_caught(monkeypatch):
    real_sort = torch.sort

    def flipped(x, stable=False, **kw):
        r = real_sort(x.flip(0), stable=True)
        return torch.return_types.sort((r.values, x.shape[0] - 1 - r.indices))
    monkeypatch.setattr(O.torch, "sort", flipped)
    try:
        assert _caught(pins.test_select_blocks_ties_and_padding)
    finally:
        monkeypatch.setattr(O.torch, "sort", real_sort)


def test_window_too_wide_is_caught(monkeypatch):
    monkeypatch.setattr(O, "window_tokens", lambda t, w: torch.arange(max(0, t - w), t + 1))
    assert _caught(pins.test_window_of_T_equals_full_causal_and_window_one_is_v)


def test_missing_scale_is_caught(monkeypatch):
    real = O.attend
    monkeypatch.setattr(O, "attend", lambda Q, K, V, scale: real(Q, K, V, 1.0))
    assert _caught(pins.test_attend_matches_sdpa, pins.test_all_blocks_selected_equals_full_causal)


def test_swapped_gates_are_caught(monkeypatch):
    real = O.nsa_token

    def bad(Qg, K, V, Kc, Vc, gates_g, t, **kw):
        return real(Qg, K, V, Kc, Vc, gates_g[:, [1, 0, 2]], t, **kw)
    monkeypatch.setattr(O, "nsa_token", bad)
    assert _caught(pins.test_gates_zero_and_one_hot, pins.test_nsa_handworked_closed_forms)


def test_future_token_in_selected_block_is_caught(monkeypatch):
    def bad(idx, t, b):      # reads one token past the query
        toks = [torch.arange(b * j, min(b * j + b, t + 2)) for j in idx if j >= 0]
        return torch.cat(toks)
    monkeypatch.setattr(O, "block_tokens", bad)
    assert _caught(pins.test_causality_future_tokens_do_not_matter)


def test_moba_without_own_block_is_caught(monkeypatch):
    real = O.moba_select

    def bad(qt, kbar, t, block, top_k):
        sel = [j for j in real(qt, kbar, t, block, top_k) if j != t // block]
        return sel + [-1] * (top_k + 1 - len(sel))
    monkeypatch.setattr(O, "moba_select", bad)
    assert _caught(pins.test_moba_handworked_closed_forms)


def test_moba_scaled_block_scores_do_not_matter_but_wrong_sign_is_caught(monkeypatch):
    real = O.moba_select
    monkeypatch.setattr(O, "moba_select", lambda qt, kbar, t, block, top_k: real(-qt, kbar, t, block, top_k))
    assert _caught(pins.test_moba_handworked_closed_forms)
