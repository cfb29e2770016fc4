"""fp64 CPU oracle for the token-wise sparse attention of DSA (DeepSeek Sparse Attention).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import or run this file; the library never calls
it and shares no code with it.

Page cited: 10100.com, "机器之心PRO · 会员通讯 Week 45", item 1 ("Which
Attention is All You Need?"), section "Linear v.s. Sparse，主流 Attention 改良
「玩」 法有哪些？", point 6.  It describes DSA in prose only: a lightweight
"Lightning Indexer" scans all tokens (O(N) per token) and gives each one an
importance proxy score; "Top-k Token Selection" keeps the k highest; full
attention runs over those k tokens.  The page gives no formula, so the
plainest readings are taken:

  D1  indexer score of key s for query t (s <= t): sum over the indexer heads
      j of w[t, j] * ReLU(q_I[t, j] . k_I[s]); q_I [T, H_I, d_I], k_I [T, d_I]
      (one key per token, shared by the indexer heads) and w [T, H_I] are
      inputs.
  D2  top-k over the keys s <= t by score, higher first, ties to the lower
      index; the list is ascending and -1 padded; with t + 1 <= k every key.
  D3  one selection per query token, shared by all its query heads.
  D4  per query head, softmax attention with scale 1/sqrt(d_k) over the
      selected tokens, the KV head of the head's GQA group.
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64


def indexer_scores(q_i: torch.Tensor, k_i: torch.Tensor, w_i: torch.Tensor, t: int) -> torch.Tensor:
    """D1 for one query token t: q_i [H_I, d_I], k_i [>= t+1, d_I], w_i [H_I] -> [t + 1]."""
    dots = k_i[: t + 1].to(F64) @ q_i.to(F64).T          # [t+1, H_I]
    return torch.relu(dots) @ w_i.to(F64)


def select_tokens(score: torch.Tensor, k: int) -> list[int]:
    """D2: the k best keys (score desc, index asc), returned ascending."""
    n = score.shape[0]
    if n <= k:
        return list(range(n))
    order = sorted(range(n), key=lambda s: (-float(score[s]), s))
    return sorted(order[:k])


def attend(qh: torch.Tensor, K: torch.Tensor, V: torch.Tensor, scale: float) -> torch.Tensor:
    """Softmax attention of query rows qh [G, d_k] over K [n, d_k], V [n, d_v] (fp64)."""
    s = (qh @ K.T) * scale
    p = torch.softmax(s, dim=-1)
    return p @ V


def dsa_forward(q, k, v, q_i, k_i, w_i, *, top_k=2048, scale=None, tokens=None, forced_idx=None):
    """DSA forward over the query positions ``tokens`` (all by default).

    q [B,T,H_q,d_k], k [B,T,H_kv,d_k], v [B,T,H_kv,d_v]; q_i [B,T,H_I,d_I],
    k_i [B,T,d_I], w_i [B,T,H_I].  ``forced_idx`` [B, n, top_k] (-1 padded)
    imposes the chosen tokens (forced-index mode: the attention over a choice
    that differs from the oracle's only at a near tie).
    Returns dict(out [B, n, H_q, d_v] fp64,
    idx [B, n, top_k] (-1 padded), score: list per (b, token) of the indexer
    scores, for the near-tie rule)."""
    q, k, v = q.to(F64), k.to(F64), v.to(F64)
    B, T, Hq, dk = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    toks = list(range(T)) if tokens is None else [int(t) for t in tokens]
    out = torch.zeros((B, len(toks), Hq, dv), dtype=F64)
    idx = torch.full((B, len(toks), top_k), -1, dtype=torch.long)
    scores = [[None] * len(toks) for _ in range(B)]
    for b in range(B):
        for n, t in enumerate(toks):
            sc = indexer_scores(q_i[b, t], k_i[b], w_i[b, t], t)
            if forced_idx is None:
                sel = select_tokens(sc, top_k)
            else:
                sel = [int(j) for j in forced_idx[b, n] if j >= 0]
            scores[b][n] = sc
            idx[b, n, : len(sel)] = torch.tensor(sel)
            rows = torch.tensor(sel)
            for g in range(Hkv):
                hs = slice(g * G, (g + 1) * G)
                out[b, n, hs] = attend(q[b, t, hs], k[b, rows, g], v[b, rows, g], scale)
    return dict(out=out, idx=idx, score=scores, tokens=toks)
