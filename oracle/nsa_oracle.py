"""fp64 CPU oracle for the Native Sparse Attention (NSA) forward pass, its
one-token decode step, and the MoBA mode.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this file.
The library itself never calls it and shares no code with it: every
function here is a plain restatement of what the method computes, written
to be checked against the pages by eye, not to be fast.

Pages cited (by title, then section):
  [NOTES] zjai.club episode notes, "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文
          （含投屏版）——“硬件上的暴力美学”", numbered sections 5-10 and 14-17.
  [EN]    youtublog.net/en, "Songlin Yang Explains Attention Mechanisms from
          DeepSeek, Kimi, and MiniMax" (paragraphs on the three branches, on
          GQA and on MoBA).
  [BLOG]  sunshychen.top, "一文比较 Kimi 和 Deepseek 的两篇稀疏注意力机制论文",
          sections "Kimi 的论文核心点" and "Deepseek 的论文核心点".

The pages give the method only in prose (their formulas did not survive).
Where they leave a step open, the plainest reading is taken; each reading is
listed as R1..R14 in the docstring of the function that applies it:

  R1  phi is a linear map (no bias) of the token-major flattened l x d block,
      one matrix for K and one for V, shared by all heads.
  R2  compressed block i is visible to query t iff its last token
      s*i + l - 1 <= t; with none visible the compressed output is 0.
  R3  the score of 64-token selection block j is the sum of the probabilities
      of every visible compressed block whose span [s*i, s*i+l) intersects
      [b*j, b*j+b) ("parity unpinned": the pages fix no mapping when the
      block sizes differ).  The two other readings are kept as options:
      "contained" (only the compressed blocks that lie inside one selection
      block count) and "overlap" (each counts with the fraction of its span
      inside the selection block).
  R4  the group sums post-softmax probabilities (each head normalised over
      its own visible compressed blocks).
  R5  block 0 and the query's own block are always selected and count toward
      k; with k or fewer eligible blocks all are taken; -1 pads the list.
  R6  top-k orders by score, higher first, ties to the lower block index;
      the emitted list is ascending.
  R7  one softmax over all tokens of the selected blocks that are <= t.
  R8  the window is the last w tokens including t.
  R9  the branches are combined by a gated sum (gates are inputs).
  R10 scale 1/sqrt(d_k) in every attention; MoBA block scoring is unscaled.
  R11 decode: the cache includes the new token, whose position is L-1.
  R12 MoBA: candidates are the complete past blocks j < t//B; block key is
      the mean of the block's keys; top-k past blocks plus the own block.
  R14 compressed K/V are stored as bf16 tensors (like every K/V tensor of the
      method); ``round_kc=True`` rounds phi's output accordingly.
  R15 phi as an MLP (an option; [BLOG] "Deepseek 的论文核心点" says the blocks are
      compressed by an MLP): two layers of hidden width d with GELU between,
      a bias on the first layer, hidden values stored in bf16.  An intra-block
      position embedding added before the first layer is that bias.
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64


def _f64(x: torch.Tensor) -> torch.Tensor:
    """fp64 on the CPU; an fp64 CPU tensor that requires grad is kept as is (autograd)."""
    if x.requires_grad and x.dtype == F64 and x.device.type == "cpu":
        return x
    return x.detach().to("cpu", F64)


def round_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round to the nearest bf16 (ties to even) and return fp64."""
    return x.to(torch.bfloat16).to(F64)


# --------------------------------------------------------------------------
# a1: block compression phi
# --------------------------------------------------------------------------

def num_cmp_blocks(T: int, l: int, s: int) -> int:
    """Number of compressed blocks of a length-T sequence: windows of l tokens
    taken every s tokens that fit entirely inside the sequence."""
    return 0 if T < l else (T - l) // s + 1


def num_visible_cmp_blocks(t: int, l: int, s: int, n_total: int) -> int:
    """R2: compressed block i is visible to query t iff s*i + l - 1 <= t."""
    if t < l - 1:
        return 0
    return min(n_total, (t - l + 1) // s + 1)


def phi_compress(X: torch.Tensor, W: torch.Tensor, l: int, s: int) -> torch.Tensor:
    """Compress one sequence of one KV head.

    [NOTES] §5: each contiguous KV block becomes one key and one value
    vector; [BLOG] "Deepseek 的论文核心点": a learned map compresses each block
    into a short k, v.  R1: row i is vec(X[s*i : s*i+l]) @ W with the block
    flattened token-major (element (r, c) at index r*d + c).

    X: [T, d]; W: [l*d, d_out] -> [N_c, d_out] (fp64)."""
    X = _f64(X)
    W = _f64(W)
    T, d = X.shape
    n = num_cmp_blocks(T, l, s)
    if n == 0:
        return torch.zeros((0, W.shape[1]), dtype=F64)
    blocks = torch.stack([X[s * i: s * i + l].reshape(l * d) for i in range(n)])
    return blocks @ W


def gelu(x: torch.Tensor) -> torch.Tensor:
    """GELU with the exact normal CDF: x * (1 + erf(x / sqrt(2))) / 2."""
    return 0.5 * x * (1.0 + torch.erf(x / math.sqrt(2.0)))


def phi_mlp(X: torch.Tensor, W1: torch.Tensor, b1: torch.Tensor, W2: torch.Tensor, l: int, s: int,
            round_hidden: bool = True) -> torch.Tensor:
    """R15: phi as a two-layer MLP of one sequence and KV head.

    Row i is GELU(vec(X[s*i : s*i+l]) @ W1 + b1) @ W2, the hidden values rounded
    to bf16 where the library stores them (``round_hidden``).

    X: [T, d]; W1: [l*d, h]; b1: [h]; W2: [h, d_out] -> [N_c, d_out] (fp64)."""
    hidden = gelu(phi_compress(X, W1, l, s) + _f64(b1))
    if round_hidden:
        hidden = round_bf16(hidden)
    return hidden @ _f64(W2)


def compress_cache(K: torch.Tensor, W: torch.Tensor, l: int, s: int,
                   round_kc: bool = True, mlp=None) -> torch.Tensor:
    """phi over every (batch, KV head): K [B, T, H, d] -> [B, N_c, H, d_out].
    ``mlp`` = (b1, W2) makes phi the two-layer MLP of R15 with W as its first layer."""
    B, T, H, _ = K.shape
    n = num_cmp_blocks(T, l, s)
    d_out = W.shape[1] if mlp is None else mlp[1].shape[1]
    out = torch.zeros((B, n, H, d_out), dtype=F64)
    for b in range(B):
        for h in range(H):
            if mlp is None:
                out[b, :, h] = phi_compress(K[b, :, h], W, l, s)
            else:
                out[b, :, h] = phi_mlp(K[b, :, h], W, mlp[0], mlp[1], l, s, round_hidden=round_kc)
    return round_bf16(out) if round_kc else out


# --------------------------------------------------------------------------
# softmax attention of a few query rows over an explicit key set
# --------------------------------------------------------------------------

def attend(Q: torch.Tensor, Kx: torch.Tensor, Vx: torch.Tensor, scale: float):
    """Plain softmax attention: rows of Q over the rows of Kx/Vx.

    Returns (o [G, d_v], p [G, n]).  With no keys the output is zero
    (the branch contributes nothing)."""
    G = Q.shape[0]
    n = Kx.shape[0]
    if n == 0:
        return torch.zeros((G, Vx.shape[1]), dtype=F64), torch.zeros((G, 0), dtype=F64)
    logits = scale * (Q @ Kx.T)
    p = torch.softmax(logits, dim=1)
    return p @ Vx, p


# --------------------------------------------------------------------------
# a2-a5 for one query token and one GQA group
# --------------------------------------------------------------------------

SCORE_MAPS = ("touch", "contained", "overlap")   # the library's NSA_MAP_* order


def selection_scores(p_cmp: torch.Tensor, t: int, l: int, s: int, b: int,
                     mapping: str = "touch") -> torch.Tensor:
    """a3, block importance for the selection branch.

    [BLOG] "Deepseek 的论文核心点": the selection scores come straight from the
    compressed attention.  [NOTES] §8: the heads of one GQA group add their
    block-selection scores before one shared top-k.  R3/R4: every visible
    compressed block i adds its probability (summed over the group's heads)
    to each selection block j whose span [b*j, b*j+b) meets [s*i, s*i+l),
    with weight 1 ("touch"); 1 if the span lies inside block j alone, else 0
    ("contained"); or the fraction of the span inside block j ("overlap").

    p_cmp: [G, n_vis] -> scores [t//b + 1]."""
    if mapping not in SCORE_MAPS:
        raise ValueError(mapping)
    nb = t // b + 1
    score = torch.zeros(nb, dtype=F64)
    if p_cmp.shape[1] == 0:
        return score
    per_block = p_cmp.sum(dim=0)                       # group sum
    i = torch.arange(per_block.shape[0])
    start, end = s * i, s * i + l                       # span [start, end)
    first = start // b                                  # first selection block touched
    last = (end - 1) // b                               # last selection block touched
    for off in range(int((last - first).max()) + 1):
        j = first + off
        hit = j <= last
        if mapping == "touch":
            w = torch.ones_like(per_block)
        elif mapping == "contained":
            w = (first == last).to(F64)
        else:
            inside = torch.minimum(end, b * (j + 1)) - torch.maximum(start, b * j)
            w = inside.to(F64) / l
        score.index_add_(0, j[hit], (w * per_block)[hit])
    return score


def select_blocks(score: torch.Tensor, t: int, b: int, k: int,
                  force_first: bool = True, force_local: bool = True) -> list[int]:
    """a3, top-k block choice for query t.  [NOTES] §5 (top-k blocks) and §8
    (one choice per group).  R5: forced blocks count toward k; R6: higher
    score first, ties to the lower index; the list is ascending, -1 padded."""
    nb = t // b + 1
    forced = []
    if force_first:
        forced.append(0)
    if force_local and (t // b) not in forced:
        forced.append(t // b)
    if nb <= k:
        chosen = list(range(nb))
    else:
        rest = torch.tensor([j for j in range(nb) if j not in forced], dtype=torch.long)
        order = torch.sort(-score[rest], stable=True).indices   # stable: ties keep lower j first
        chosen = forced + rest[order[: k - len(forced)]].tolist()
    chosen = sorted(chosen)
    return chosen + [-1] * (k - len(chosen))


def block_tokens(idx: list[int], t: int, b: int) -> torch.Tensor:
    """R7: all tokens of the selected blocks that are not in the future."""
    toks = [torch.arange(b * j, min(b * j + b, t + 1)) for j in idx if j >= 0]
    toks = [x for x in toks if x.numel()]
    return torch.cat(toks) if toks else torch.zeros(0, dtype=torch.long)


def window_tokens(t: int, w: int) -> torch.Tensor:
    """R8: the last w tokens up to and including t ([NOTES] §5, sliding window)."""
    return torch.arange(max(0, t - w + 1), t + 1)


def nsa_token(Qg, K, V, Kc, Vc, gates_g, t, *, l, s, b, k, w, scale,
              force_first=True, force_local=True, idx=None, score_map="touch"):
    """All three branches of one query token for one GQA group.

    Qg: [G, d_k] the group's query rows; K, V: [>=t+1, d] this KV head's
    keys/values; Kc, Vc: [N_c, d] its compressed keys/values; gates_g: [G, 3].
    [NOTES] §5-§6: compressed, selected and sliding-window attention, each
    weighted by a per-token gate and summed (R9).
    Returns dict(out, o_cmp, o_slc, o_win, idx, score)."""
    n_vis = num_visible_cmp_blocks(t, l, s, Kc.shape[0])
    o_cmp, p_cmp = attend(Qg, Kc[:n_vis], Vc[:n_vis], scale)          # a2
    score = selection_scores(p_cmp, t, l, s, b, score_map)           # a3
    if idx is None:
        idx = select_blocks(score, t, b, k, force_first, force_local)
    sel = block_tokens(idx, t, b)
    o_slc, _ = attend(Qg, K[sel], V[sel], scale)                      # a4
    win = window_tokens(t, w)
    o_win, _ = attend(Qg, K[win], V[win], scale)                      # a5
    out = gates_g[:, 0:1] * o_cmp + gates_g[:, 1:2] * o_slc + gates_g[:, 2:3] * o_win   # a6
    return dict(out=out, o_cmp=o_cmp, o_slc=o_slc, o_win=o_win, idx=idx, score=score)


# --------------------------------------------------------------------------
# a1-a6: prefill forward
# --------------------------------------------------------------------------

def nsa_forward(q, k, v, gates, w_k, w_v, *, cmp_block=32, cmp_stride=16,
                sel_block=64, top_k=16, window=512, force_first=True,
                force_local=True, scale=None, tokens=None, round_kc=True,
                keep_branches=False, score_map="touch", mlp=None, forced_idx=None):
    """NSA prefill forward over the query positions ``tokens`` (all by default).

    q [B,T,H_q,d_k], k [B,T,H_kv,d_k], v [B,T,H_kv,d_v], gates [B,T,H_q,3],
    w_k [l*d_k,d_k], w_v [l*d_v,d_v].  Query head h belongs to group
    h // (H_q // H_kv) ([EN], GQA paragraph; [NOTES] §7).

    ``mlp`` = dict(b_k, w_k2, b_v, w_v2) makes phi the two-layer MLP of R15
    (w_k, w_v are then its first layers); ``score_map`` picks the R3 reading;
    ``forced_idx`` [B, H_kv, n_tok, top_k] imposes the chosen blocks (forced-index mode).
    The function is differentiable (torch autograd) in q, k, v, gates, w_k, w_v
    given fp64 leaf tensors; the block choice is discrete.

    Returns a dict with fp64 ``out`` [B, n_tok, H_q, d_v], int ``idx``
    [B, H_kv, n_tok, top_k], ``score`` (list per (b, g, token) of the block
    scores, for the near-tie rule), ``kc``/``vc`` and, if asked, the three
    branch outputs."""
    q, k, v, gates = _f64(q), _f64(k), _f64(v), _f64(gates)
    B, T, Hq, dk = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    G = Hq // Hkv
    l, s, b = cmp_block, cmp_stride, sel_block
    scale = 1.0 / math.sqrt(dk) if scale is None else scale                 # R10
    toks = list(range(T)) if tokens is None else [int(t) for t in tokens]
    kc = compress_cache(k, w_k, l, s, round_kc, None if mlp is None else (mlp["b_k"], mlp["w_k2"]))
    vc = compress_cache(v, w_v, l, s, round_kc, None if mlp is None else (mlp["b_v"], mlp["w_v2"]))
    n = len(toks)
    out = torch.zeros((B, n, Hq, dv), dtype=F64)
    idx = torch.full((B, Hkv, n, top_k), -1, dtype=torch.long)
    branches = {name: torch.zeros((B, n, Hq, dv), dtype=F64)
                for name in ("o_cmp", "o_slc", "o_win")} if keep_branches else None
    scores = [[[None] * n for _ in range(Hkv)] for _ in range(B)]
    for bi in range(B):
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            for n_i, t in enumerate(toks):
                r = nsa_token(q[bi, t, hs], k[bi, :, g], v[bi, :, g], kc[bi, :, g], vc[bi, :, g],
                              gates[bi, t, hs], t, l=l, s=s, b=b, k=top_k, w=window,
                              scale=scale, force_first=force_first, force_local=force_local,
                              score_map=score_map,
                              idx=None if forced_idx is None else [int(j) for j in forced_idx[bi, g, n_i]])
                out[bi, n_i, hs] = r["out"]
                idx[bi, g, n_i] = torch.tensor(r["idx"])
                scores[bi][g][n_i] = r["score"]
                if keep_branches:
                    for name in branches:
                        branches[name][bi, n_i, hs] = r[name]
    res = dict(out=out, idx=idx, score=scores, kc=kc, vc=vc, tokens=toks)
    if keep_branches:
        res.update(branches)
    return res


# --------------------------------------------------------------------------
# a7: decode (one new query per sequence)
# --------------------------------------------------------------------------

def nsa_decode(q, k_cache, v_cache, kc_cache, vc_cache, seqlens, gates, *,
               cmp_block=32, cmp_stride=16, sel_block=64, top_k=16, window=512,
               force_first=True, force_local=True, scale=None, batch=None, score_map="touch",
               forced_idx=None):
    """One decode step.  [NOTES] §13: decoding reads the KV cache once per
    step; R11: sequence b's cache holds seqlens[b] tokens including the new
    one, whose position is t = seqlens[b] - 1.  The compressed caches are
    inputs (the compressed blocks visible to t are exactly those of a
    length-seqlens[b] sequence).

    q [B,H_q,d_k], caches [B,L,H_kv,d], kc/vc [B,N_c,H_kv,d], gates [B,H_q,3].
    ``batch`` restricts the work to some sequences.  ``forced_idx`` [nb, H_kv, top_k] (one
    row per sequence worked on) imposes the chosen blocks (forced-index mode).
    Returns dict(out [nb, H_q, d_v], idx [nb, H_kv, top_k], score)."""
    q, gates = _f64(q), _f64(gates)
    B, Hq, dk = q.shape
    Hkv = k_cache.shape[2]
    dv = v_cache.shape[3]
    G = Hq // Hkv
    l, s, b = cmp_block, cmp_stride, sel_block
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    bs = list(range(B)) if batch is None else list(batch)
    out = torch.zeros((len(bs), Hq, dv), dtype=F64)
    idx = torch.full((len(bs), Hkv, top_k), -1, dtype=torch.long)
    scores = []
    for n_i, bi in enumerate(bs):
        L = int(seqlens[bi])
        t = L - 1
        nc = num_cmp_blocks(L, l, s)
        row = []
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            r = nsa_token(q[bi, hs], _f64(k_cache[bi, :L, g]), _f64(v_cache[bi, :L, g]),
                          _f64(kc_cache[bi, :nc, g]), _f64(vc_cache[bi, :nc, g]),
                          gates[bi, hs], t, l=l, s=s, b=b, k=top_k, w=window, scale=scale,
                          force_first=force_first, force_local=force_local, score_map=score_map,
                          idx=None if forced_idx is None else [int(j) for j in forced_idx[n_i, g]])
            out[n_i, hs] = r["out"]
            idx[n_i, g] = torch.tensor(r["idx"])
            row.append(r["score"])
        scores.append(row)
    return dict(out=out, idx=idx, score=scores)


# --------------------------------------------------------------------------
# a8: MoBA mode
# --------------------------------------------------------------------------

def moba_block_keys(K: torch.Tensor, block: int) -> torch.Tensor:
    """[NOTES] §16; [BLOG] "Kimi 的论文核心点": each block is represented by the
    mean of its keys (mean pooling, no parameters).  K: [T, d] -> [ceil(T/B), d]."""
    K = _f64(K)
    T, d = K.shape
    nb = (T + block - 1) // block
    return torch.stack([K[j * block: min(T, (j + 1) * block)].mean(dim=0) for j in range(nb)])


def moba_select(qt: torch.Tensor, kbar: torch.Tensor, t: int, block: int, top_k: int) -> list[int]:
    """R12: score_j = q . mean(K_j) over the complete past blocks j < t//B
    (unscaled, R10); the top_k of them (ties to the lower index) plus the own
    block t//B, which is always attended ([BLOG] "Kimi 的论文核心点").
    Ascending list, -1 padded to top_k + 1."""
    own = t // block
    if own <= top_k:
        chosen = list(range(own))
    else:
        sc = kbar[:own] @ qt
        chosen = torch.sort(-sc, stable=True).indices[:top_k].tolist()
    chosen = sorted(chosen) + [own]
    return chosen + [-1] * (top_k + 1 - len(chosen))


def moba_forward(q, k, v, *, block=512, top_k=3, scale=None, tokens=None, heads=None, forced_idx=None):
    """MoBA forward: per head, softmax attention over the tokens (<= t) of
    the chosen past blocks and of the own block (causal inside it).
    [BLOG] "Kimi 的论文核心点": selecting every block gives full attention,
    selecting none leaves only the own block.

    q, k, v: [B, T, H, d].  ``forced_idx`` [B, H, n_tok, top_k+1] imposes the
    chosen blocks (forced-index mode, as in ``nsa_forward``: where two block
    choices are equally correct up to a near tie, the output is checked for
    the choice actually made).  Returns dict(out [B, n_tok, H, d], idx
    [B, H, n_tok, top_k+1], score list for the near-tie rule)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    toks = list(range(T)) if tokens is None else [int(t) for t in tokens]
    hl = list(range(H)) if heads is None else list(heads)
    n = len(toks)
    out = torch.zeros((B, n, H, d), dtype=F64)
    idx = torch.full((B, H, n, top_k + 1), -1, dtype=torch.long)
    scores = {}
    for bi in range(B):
        for h in hl:
            kbar = moba_block_keys(k[bi, :, h], block)
            for n_i, t in enumerate(toks):
                if forced_idx is None:
                    sel = moba_select(q[bi, t, h], kbar, t, block, top_k)
                else:
                    sel = [int(j) for j in forced_idx[bi, h, n_i]]
                toks_u = block_tokens(sel, t, block)
                o, _ = attend(q[bi, t, h:h + 1], k[bi, toks_u, h], v[bi, toks_u, h], scale)
                out[bi, n_i, h] = o[0]
                idx[bi, h, n_i] = torch.tensor(sel)
                own = t // block
                scores[(bi, h, n_i)] = kbar[:own] @ q[bi, t, h]
    return dict(out=out, idx=idx, score=scores, tokens=toks)
