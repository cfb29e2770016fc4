"""The comparison rules of the GPU parity tests, checked on the CPU: the near-tie rule for
block choices rejects a choice that leaves out a clearly better block, and the oracle's
forced-index modes reproduce the oracle's own output when given its own choice."""
import pytest
import torch

import oracle
import synth
from tests.helpers import NEAR_TIE, check_swap, idx_agreement, with_forced_rows


def _one_token(choice, oracle_choice, score, t=640):
    k = len(oracle_choice)
    pad = lambda c: sorted(c) + [-1] * (k - len(c))
    gpu = torch.tensor([[[pad(choice)]]])
    ora = torch.tensor([[[pad(oracle_choice)]]])
    return idx_agreement(gpu, ora, [[[score]]], tokens=[t])


def test_legal_near_tie_swap_is_accepted():
    score = torch.zeros(11, dtype=torch.float64)
    score[3], score[5], score[7] = 10.0, 1.0, 1.0 - NEAR_TIE / 2
    exact, swapped = _one_token([0, 3, 7, 10], [0, 3, 5, 10], score)
    assert exact == 0 and swapped == {(0, 0, 0)}


def test_dropping_a_clearly_best_block_is_rejected():
    """The oracle picks a block scoring 10 and one at the k-th score 1.0; a GPU set that drops
    the 10 and adds a block scoring just under 1.0 is not a near-tie swap."""
    score = torch.zeros(11, dtype=torch.float64)
    score[3], score[5], score[7] = 10.0, 1.0, 1.0 - NEAR_TIE / 2
    with pytest.raises(AssertionError):
        _one_token([0, 5, 7, 10], [0, 3, 5, 10], score)


def test_adding_a_clearly_worse_block_is_rejected():
    score = torch.zeros(11, dtype=torch.float64)
    score[3], score[5], score[7] = 10.0, 1.0, 0.5
    with pytest.raises(AssertionError):
        _one_token([0, 3, 7, 10], [0, 3, 5, 10], score)


def test_missing_forced_block_and_wrong_count_are_rejected():
    score = torch.ones(11, dtype=torch.float64)
    with pytest.raises(AssertionError):
        _one_token([1, 3, 5, 10], [0, 3, 5, 10], score)      # block 0 is forced
    with pytest.raises(AssertionError):
        _one_token([0, 3, 10], [0, 3, 5, 10], score)         # one block short


def test_check_swap_without_fixed_blocks():
    score = [5.0, 4.0, 3.0, 3.0 - 1e-4, 1.0]
    check_swap([0, 1, 3], [0, 1, 2], score, (), 1e-3)
    with pytest.raises(AssertionError):
        check_swap([0, 2, 3], [0, 1, 2], score, (), 1e-3)


def test_forced_rows_replace_only_swapped_positions():
    ref = torch.zeros(1, 4, 2)
    out = with_forced_rows(ref, {(0, 0, 1), (0, 1, 3)}, lambda pos: torch.full((1, len(pos), 2), float(len(pos))))
    assert out[0, 0].eq(0).all() and out[0, 2].eq(0).all()
    assert out[0, 1].eq(2).all() and out[0, 3].eq(2).all()
    assert ref.eq(0).all()


def test_nsa_forced_index_mode_with_own_choice_reproduces_the_oracle():
    x = synth.nsa_inputs(1, 300, 8, 2, 64, 64, seed=90)
    toks = [0, 70, 199, 299]
    ref = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=3, window=50, tokens=toks)
    again = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=3, window=50, tokens=toks,
                               forced_idx=ref["idx"])
    assert torch.equal(ref["out"], again["out"])
    other = ref["idx"].clone()
    other[0, 0, 3] = torch.tensor([0, 2, 4])             # a different (valid) choice for t = 299
    moved = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=3, window=50, tokens=toks,
                               forced_idx=other)
    assert torch.equal(moved["out"][:, :3], ref["out"][:, :3])
    assert not torch.allclose(moved["out"][0, 3, :4], ref["out"][0, 3, :4])


def test_moba_forced_index_mode_with_own_choice_reproduces_the_oracle():
    x = synth.moba_inputs(1, 400, 2, 16, seed=91)
    ref = oracle.moba_forward(x.q, x.k, x.v, block=64, top_k=2, tokens=[10, 200, 399])
    again = oracle.moba_forward(x.q, x.k, x.v, block=64, top_k=2, tokens=[10, 200, 399], forced_idx=ref["idx"])
    assert torch.equal(ref["out"], again["out"])


def test_dsa_forced_index_mode_with_own_choice_reproduces_the_oracle():
    x = synth.dsa_inputs(1, 90, 4, 1, 64, 64, 2, 64, seed=92)
    toks = [3, 40, 89]
    ref = oracle.dsa_forward(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w_idx, top_k=16, tokens=toks)
    again = oracle.dsa_forward(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w_idx, top_k=16, tokens=toks,
                               forced_idx=ref["idx"])
    assert torch.equal(ref["out"], again["out"])


def test_decode_forced_index_mode_with_own_choice_reproduces_the_oracle():
    d = synth.decode_inputs(2, 400, 8, 2, 64, 64, seed=93)
    sl = torch.tensor([400, 257], dtype=torch.int32)
    kc = oracle.compress_cache(d.k_cache, d.w_k, 32, 16)
    vc = oracle.compress_cache(d.v_cache, d.w_v, 32, 16)
    run = lambda forced=None, batch=None: oracle.nsa_decode(d.q, d.k_cache, d.v_cache, kc, vc, sl, d.gates,
                                                            top_k=3, window=50, batch=batch, forced_idx=forced)
    ref = run()
    assert torch.equal(run(ref["idx"])["out"], ref["out"])
    assert torch.equal(run(ref["idx"][1:], batch=[1])["out"], ref["out"][1:])
    other = ref["idx"].clone()
    other[0, 1] = torch.tensor([0, 1, 6])                 # another valid choice for sequence 0, group 1
    moved = run(other)["out"]
    assert torch.equal(moved[1], ref["out"][1]) and torch.equal(moved[0, :4], ref["out"][0, :4])
    assert not torch.allclose(moved[0, 4:], ref["out"][0, 4:])
