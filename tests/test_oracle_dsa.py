"""Pins of the DSA oracle (token-wise sparse attention behind a lightning indexer) against
closed forms, brute force and library routines."""
import math

import torch
import torch.nn.functional as F

import oracle


def test_indexer_closed_form():
    """One head, weight 2: the score is 2 * ReLU(q . k_s); negative dots give 0."""
    q = torch.tensor([[1.0, -2.0]], dtype=torch.float64)
    k = torch.tensor([[3.0, 1.0], [0.0, 1.0], [2.0, 0.5]], dtype=torch.float64)
    w = torch.tensor([2.0], dtype=torch.float64)
    assert oracle.indexer_scores(q, k, w, 2).tolist() == [2.0, 0.0, 2.0]
    assert oracle.indexer_scores(q, k, w, 0).tolist() == [2.0]


def test_indexer_heads_add_with_their_weights():
    g = torch.Generator().manual_seed(1)
    q = torch.randn(3, 8, generator=g, dtype=torch.float64)
    k = torch.randn(10, 8, generator=g, dtype=torch.float64)
    w = torch.tensor([0.5, -1.0, 2.0], dtype=torch.float64)
    want = sum(w[j] * torch.clamp(k @ q[j], min=0) for j in range(3))
    assert torch.allclose(oracle.indexer_scores(q, k, w, 9), want, atol=1e-14, rtol=0)


def test_select_tokens_matches_a_full_sort_with_ties():
    score = torch.tensor([3.0, 1.0, 3.0, 2.0, 3.0, 0.0], dtype=torch.float64)
    assert oracle.select_tokens(score, 2) == [0, 2]          # three tie at 3.0: the lower indices
    assert oracle.select_tokens(score, 4) == [0, 2, 3, 4]
    assert oracle.select_tokens(score, 6) == list(range(6))
    assert oracle.select_tokens(score, 9) == list(range(6))
    g = torch.Generator().manual_seed(2)
    s = torch.randint(0, 5, (40,), generator=g).to(torch.float64)
    ref = sorted(sorted(range(40), key=lambda i: (-float(s[i]), i))[:11])
    assert oracle.select_tokens(s, 11) == ref


def test_all_tokens_selected_is_full_causal_attention():
    """top_k >= T: every token attends to all earlier ones (SDPA with a causal mask)."""
    g = torch.Generator().manual_seed(3)
    B, T, Hq, Hkv, dk, dv, HI, dI = 1, 24, 4, 2, 8, 6, 2, 4
    q = torch.randn(B, T, Hq, dk, generator=g, dtype=torch.float64)
    k = torch.randn(B, T, Hkv, dk, generator=g, dtype=torch.float64)
    v = torch.randn(B, T, Hkv, dv, generator=g, dtype=torch.float64)
    qi = torch.randn(B, T, HI, dI, generator=g, dtype=torch.float64)
    ki = torch.randn(B, T, dI, generator=g, dtype=torch.float64)
    wi = torch.randn(B, T, HI, generator=g, dtype=torch.float64)
    r = oracle.dsa_forward(q, k, v, qi, ki, wi, top_k=T)
    kk = k.repeat_interleave(Hq // Hkv, dim=2).transpose(1, 2)
    vv = v.repeat_interleave(Hq // Hkv, dim=2).transpose(1, 2)
    ref = F.scaled_dot_product_attention(q.transpose(1, 2), kk, vv, is_causal=True).transpose(1, 2)
    assert torch.allclose(r["out"], ref, atol=1e-12, rtol=0)


def test_selection_and_future_tokens():
    """The selected set holds top_k tokens <= t; changing tokens after t changes nothing."""
    g = torch.Generator().manual_seed(4)
    B, T, Hq, Hkv, dk, dv, HI, dI, K = 1, 40, 2, 1, 8, 8, 2, 4, 5
    args = [torch.randn(B, T, Hq, dk, generator=g, dtype=torch.float64),
            torch.randn(B, T, Hkv, dk, generator=g, dtype=torch.float64),
            torch.randn(B, T, Hkv, dv, generator=g, dtype=torch.float64),
            torch.randn(B, T, HI, dI, generator=g, dtype=torch.float64),
            torch.randn(B, T, dI, generator=g, dtype=torch.float64),
            torch.randn(B, T, HI, generator=g, dtype=torch.float64)]
    r = oracle.dsa_forward(*args, top_k=K, tokens=[30])
    sel = r["idx"][0, 0].tolist()
    assert len(sel) == K and all(0 <= s <= 30 for s in sel) and sel == sorted(sel)
    changed = [a.clone() for a in args]
    for a in changed:
        a[:, 31:] = torch.randn(a[:, 31:].shape, generator=g, dtype=torch.float64)
    r2 = oracle.dsa_forward(*changed, top_k=K, tokens=[30])
    assert torch.equal(r["idx"], r2["idx"]) and torch.allclose(r["out"], r2["out"], atol=0, rtol=0)
    # the attention equals softmax over exactly the selected rows
    q, k, v = args[0], args[1], args[2]
    s = (q[0, 30] @ k[0, sel, 0].T) / math.sqrt(dk)
    assert torch.allclose(r["out"][0, 0], torch.softmax(s, -1) @ v[0, sel, 0], atol=1e-14, rtol=0)
