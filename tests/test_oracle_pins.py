"""Pins for the CPU oracle: each test checks it against something other than
itself -- hand-worked closed forms (tests/golden), brute force over explicit
sets, library routines (torch SDPA in fp64) for the cases the method reduces
to, and invariants the pages state.  CPU only."""
import itertools
import json
import math
import os

import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64


def closed(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e}))


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in fp64 with GQA expansion; q [T,H,d], k/v [S,Hkv,d]."""
    q, k, v = q.to(F64), k.to(F64), v.to(F64)
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1),
                                       attn_mask=mask, is_causal=causal, scale=scale)
    return o.transpose(0, 1)


# ---------------------------------------------------------------- a1: phi

def test_phi_matches_bruteforce_sum():
    g = torch.Generator().manual_seed(1)
    T, d, l, s, dout = 23, 3, 4, 2, 5
    X = torch.randn(T, d, generator=g, dtype=F64)
    W = torch.randn(l * d, dout, generator=g, dtype=F64)
    got = oracle.phi_compress(X, W, l, s)
    n = (T - l) // s + 1
    assert got.shape == (n, dout)
    for i in range(n):
        for o in range(dout):
            acc = 0.0
            for r in range(l):
                for c in range(d):
                    acc += float(X[s * i + r, c]) * float(W[r * d + c, o])
            assert abs(acc - float(got[i, o])) < 1e-12


def test_phi_selector_and_meanpool_closed_forms():
    g = torch.Generator().manual_seed(2)
    T, d, l, s = 40, 4, 8, 4
    X = torch.randn(T, d, generator=g, dtype=F64)
    for r0 in (1, l - 1):                      # W copies token r0 of each window
        W = torch.zeros(l * d, d, dtype=F64)
        for c in range(d):
            W[r0 * d + c, c] = 1.0
        got = oracle.phi_compress(X, W, l, s)
        want = torch.stack([X[s * i + r0] for i in range(got.shape[0])])
        assert torch.equal(got, want)
    W = torch.zeros(l * d, d, dtype=F64)        # mean pooling of each window
    for r in range(l):
        for c in range(d):
            W[r * d + c, c] = 1.0 / l
    got = oracle.phi_compress(X, W, l, s)
    want = torch.stack([X[s * i: s * i + l].mean(0) for i in range(got.shape[0])])
    assert torch.allclose(got, want, atol=1e-14)


@pytest.mark.parametrize("T,l,s,n", [(0, 32, 16, 0), (31, 32, 16, 0), (32, 32, 16, 1), (47, 32, 16, 1),
                                     (48, 32, 16, 2), (1024, 32, 16, 63), (8192, 32, 16, 511),
                                     (65536, 32, 16, 4095)])
def test_num_cmp_blocks(T, l, s, n):
    assert oracle.num_cmp_blocks(T, l, s) == n


def test_visible_blocks_match_definition():
    l, s = 32, 16
    n_total = oracle.num_cmp_blocks(1000, l, s)
    for t in range(1000):
        want = sum(1 for i in range(n_total) if s * i + l - 1 <= t)
        assert oracle.num_visible_cmp_blocks(t, l, s, n_total) == want


def test_compress_cache_rounds_to_bf16():
    x = synth.nsa_inputs(1, 100, 2, 1, 8, 8, cmp_block=4)
    kc = oracle.compress_cache(x.k, x.w_k, 4, 2, round_kc=True)
    exact = oracle.compress_cache(x.k, x.w_k, 4, 2, round_kc=False)
    assert torch.equal(kc, exact.to(torch.bfloat16).to(F64))
    assert (kc - exact).abs().max() <= exact.abs().max() * 2 ** -8


# ---------------------------------------------------------------- softmax attention

def test_attend_matches_sdpa():
    g = torch.Generator().manual_seed(3)
    Q = torch.randn(5, 7, generator=g, dtype=F64)
    K = torch.randn(11, 7, generator=g, dtype=F64)
    V = torch.randn(11, 3, generator=g, dtype=F64)
    o, p = oracle.attend(Q, K, V, 1 / math.sqrt(7))
    want = F.scaled_dot_product_attention(Q[None], K[None], V[None])[0]
    assert torch.allclose(o, want, atol=1e-13)
    assert torch.allclose(p.sum(1), torch.ones(5, dtype=F64), atol=1e-14)


# ---------------------------------------------------------------- hand-worked examples

def _handworked_inputs():
    cfg = json.load(open(os.path.join(GOLDEN, "nsa_handworked.json")))
    c = cfg["config"]
    T = c["T"]
    q = torch.zeros(1, T, 2, 1, dtype=F64)
    q[0, :, 0, 0] = 1.0
    k = torch.zeros(1, T, 1, 1, dtype=F64)
    k[0, 3, 0, 0] = 2.0
    k[0, 9, 0, 0] = 1.0
    v = torch.arange(T, dtype=F64).reshape(1, T, 1, 1)
    w_k = torch.tensor(cfg["inputs"]["w_k"], dtype=F64)
    w_v = torch.tensor(cfg["inputs"]["w_v"], dtype=F64)
    gates = torch.tensor(cfg["inputs"]["gates"], dtype=F64).expand(1, T, 2, 3).clone()
    return cfg, q, k, v, w_k, w_v, gates


def test_nsa_handworked_closed_forms():
    cfg, q, k, v, w_k, w_v, gates = _handworked_inputs()
    c = cfg["config"]
    toks = [e["t"] for e in cfg["expected"]]
    r = oracle.nsa_forward(q, k, v, gates, w_k, w_v, cmp_block=c["cmp_block"], cmp_stride=c["cmp_stride"],
                           sel_block=c["sel_block"], top_k=c["top_k"], window=c["window"],
                           scale=c["scale"], tokens=toks, keep_branches=True)
    g = cfg["inputs"]["gates"]
    for n, e in enumerate(cfg["expected"]):
        assert r["idx"][0, 0, n].tolist() == e["idx"], e["t"]
        for h in range(2):
            oc, os_, ow = (closed(e[name][h]) for name in ("o_cmp", "o_slc", "o_win"))
            assert abs(float(r["o_cmp"][0, n, h, 0]) - oc) < 1e-12
            assert abs(float(r["o_slc"][0, n, h, 0]) - os_) < 1e-12
            assert abs(float(r["o_win"][0, n, h, 0]) - ow) < 1e-12
            assert abs(float(r["out"][0, n, h, 0]) - (g[0] * oc + g[1] * os_ + g[2] * ow)) < 1e-12
        if "score" in e:
            sc = r["score"][0][0][n]
            assert sc.shape[0] == len(e["score"])
            for j, ex in enumerate(e["score"]):
                assert abs(float(sc[j]) - closed(ex)) < 1e-12


def test_moba_handworked_closed_forms():
    cfg = json.load(open(os.path.join(GOLDEN, "moba_handworked.json")))
    c = cfg["config"]
    T = c["T"]
    q = torch.zeros(1, T, 2, 1, dtype=F64)
    q[0, :, 0, 0] = 1.0
    q[0, :, 1, 0] = -1.0
    k = torch.zeros(1, T, 2, 1, dtype=F64)
    k[0, 3] = 4.0
    k[0, 4:8] = 0.5
    v = torch.arange(T, dtype=F64).reshape(1, T, 1, 1).expand(1, T, 2, 1).clone()
    toks = [e["t"] for e in cfg["expected"]]
    r = oracle.moba_forward(q, k, v, block=c["block"], top_k=c["top_k"], tokens=toks)
    for n, e in enumerate(cfg["expected"]):
        for h in range(2):
            assert r["idx"][0, h, n].tolist() == e["idx"][h], (e["t"], h)
            assert abs(float(r["out"][0, n, h, 0]) - closed(e["out"][h])) < 1e-12, (e["t"], h)


# ---------------------------------------------------------------- a3: scores and top-k

def test_selection_scores_match_token_set_overlap():
    """Brute force: block i contributes to block j iff their token sets share a token."""
    g = torch.Generator().manual_seed(4)
    l, s, b, G = 32, 16, 64, 3
    for t in (31, 47, 63, 64, 200, 511, 700):
        n_vis = oracle.num_visible_cmp_blocks(t, l, s, 10 ** 6)
        p = torch.rand(G, n_vis, generator=g, dtype=F64)
        got = oracle.selection_scores(p, t, l, s, b)
        want = torch.zeros(t // b + 1, dtype=F64)
        for j in range(t // b + 1):
            blk = set(range(b * j, b * j + b))
            for i in range(n_vis):
                if blk & set(range(s * i, s * i + l)):
                    for h in range(G):
                        want[j] += p[h, i]
        assert torch.allclose(got, want, atol=1e-12), t
        # the l=32/s=16/b=64 map: j collects i = 4j-1 .. 4j+3
        for j in range(t // b + 1):
            ids = [i for i in range(4 * j - 1, 4 * j + 4) if 0 <= i < n_vis]
            assert abs(float(want[j]) - float(p[:, ids].sum())) < 1e-12


def test_select_blocks_is_best_subset():
    """Brute force over every k-subset that holds the forced blocks."""
    g = torch.Generator().manual_seed(5)
    b, k = 64, 4
    for t in (64 * 7 + 5, 64 * 9, 64 * 10 - 1):
        nb = t // b + 1
        score = torch.rand(nb, generator=g, dtype=F64)
        forced = {0, t // b}
        best, best_sum = None, -1.0
        for sub in itertools.combinations(range(nb), k):
            if not forced <= set(sub):
                continue
            tot = float(sum(score[j] for j in sub if j not in forced))
            if tot > best_sum:
                best, best_sum = sorted(sub), tot
        assert oracle.select_blocks(score, t, b, k) == best


def test_select_blocks_ties_and_padding():
    b = 64
    t = 64 * 9 + 3
    score = torch.zeros(10, dtype=F64)
    assert oracle.select_blocks(score, t, b, 4) == [0, 1, 2, 9]        # ties -> lower index
    score[5] = score[7] = 1.0
    assert oracle.select_blocks(score, t, b, 4) == [0, 5, 7, 9]
    assert oracle.select_blocks(score, 100, b, 4) == [0, 1, -1, -1]    # two eligible blocks
    assert oracle.select_blocks(score, 10, b, 4) == [0, -1, -1, -1]
    assert oracle.select_blocks(score, t, b, 4, force_first=False, force_local=False) == [0, 1, 5, 7]
    s2 = torch.zeros(10, dtype=F64)
    s2[3] = 2.0
    assert oracle.select_blocks(s2, t, b, 2, force_first=False, force_local=False) == [0, 3]


# ---------------------------------------------------------------- reductions to dense attention

CFG_SMALL = dict(B=1, T=300, h_q=4, h_kv=2, d_k=16, d_v=8)


def _small(seed=0, **kw):
    c = dict(CFG_SMALL)
    c.update(kw)
    return synth.nsa_inputs(c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"], cmp_block=32, seed=seed), c


def test_all_blocks_selected_equals_full_causal():
    """Spec invariant: top-k covering every block with only the
    selection gate on is full causal attention."""
    x, c = _small()
    gates = synth.one_hot_gates(1, c["T"], c["h_q"], 1)
    r = oracle.nsa_forward(x.q, x.k, x.v, gates, x.w_k, x.w_v, top_k=c["T"] // 64 + 1, window=16)
    want = sdpa(x.q[0], x.k[0], x.v[0], causal=True)
    assert torch.allclose(r["out"][0], want, atol=1e-12)


def test_window_of_T_equals_full_causal_and_window_one_is_v():
    x, c = _small(seed=1)
    gates = synth.one_hot_gates(1, c["T"], c["h_q"], 2)
    r = oracle.nsa_forward(x.q, x.k, x.v, gates, x.w_k, x.w_v, top_k=4, window=c["T"])
    want = sdpa(x.q[0], x.k[0], x.v[0], causal=True)
    assert torch.allclose(r["out"][0], want, atol=1e-12)
    r1 = oracle.nsa_forward(x.q, x.k, x.v, gates, x.w_k, x.w_v, top_k=4, window=1)
    G = c["h_q"] // c["h_kv"]
    assert torch.allclose(r1["out"][0], x.v[0].to(F64).repeat_interleave(G, dim=1), atol=0)


def test_compressed_branch_equals_block_causal_sdpa():
    x, c = _small(seed=2)
    l, s = 32, 16
    gates = synth.one_hot_gates(1, c["T"], c["h_q"], 0)
    r = oracle.nsa_forward(x.q, x.k, x.v, gates, x.w_k, x.w_v, top_k=4, window=16)
    kc, vc = r["kc"][0], r["vc"][0]
    n = kc.shape[0]
    mask = torch.tensor([[s * i + l - 1 <= t for i in range(n)] for t in range(c["T"])])
    rows = mask.any(1)
    want = sdpa(x.q[0, rows], kc, vc, mask=mask[rows])
    assert torch.allclose(r["out"][0, rows], want, atol=1e-12)
    assert torch.equal(r["out"][0, ~rows], torch.zeros_like(r["out"][0, ~rows]))
    assert int((~rows).sum()) == l - 1


def test_gates_zero_and_one_hot():
    x, c = _small(seed=3)
    zero = torch.zeros(1, c["T"], c["h_q"], 3)
    r0 = oracle.nsa_forward(x.q, x.k, x.v, zero, x.w_k, x.w_v, top_k=3, window=40)
    assert torch.equal(r0["out"], torch.zeros_like(r0["out"]))
    r = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=3, window=40, keep_branches=True)
    for br, name in enumerate(("o_cmp", "o_slc", "o_win")):
        rb = oracle.nsa_forward(x.q, x.k, x.v, synth.one_hot_gates(1, c["T"], c["h_q"], br),
                                x.w_k, x.w_v, top_k=3, window=40)
        assert torch.equal(rb["out"], r[name])
    g = x.gates.to(F64)
    mix = g[..., 0:1] * r["o_cmp"] + g[..., 1:2] * r["o_slc"] + g[..., 2:3] * r["o_win"]
    assert torch.allclose(r["out"], mix, atol=1e-14)


def test_selection_is_shared_by_the_group_and_uses_all_heads():
    """idx carries no head index; the group sum changes the choice compared
    with any single head's own ranking on this input."""
    x, c = _small(seed=4, T=640, h_q=8, h_kv=1)
    r = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=4, window=16, tokens=range(300, 640))
    assert r["idx"].shape == (1, 1, 340, 4)
    kc, vc = r["kc"][0, :, 0], r["vc"][0, :, 0]
    differs = 0
    for n, t in enumerate(range(300, 640)):
        nv = oracle.num_visible_cmp_blocks(t, 32, 16, kc.shape[0])
        _, p = oracle.attend(x.q[0, t].to(F64), kc[:nv], vc[:nv], 1 / math.sqrt(16))
        alone = oracle.select_blocks(oracle.selection_scores(p[:1], t, 32, 16, 64), t, 64, 4)
        differs += alone != r["idx"][0, 0, n].tolist()
    assert differs > 0


def test_causality_future_tokens_do_not_matter():
    x, c = _small(seed=5)
    t0 = 170
    r = oracle.nsa_forward(x.q, x.k, x.v, x.gates, x.w_k, x.w_v, top_k=3, window=50, tokens=range(t0 + 1))
    k2, v2 = x.k.clone(), x.v.clone()
    k2[:, t0 + 1:] = 7.0
    v2[:, t0 + 1:] = -3.0
    r2 = oracle.nsa_forward(x.q, k2, v2, x.gates, x.w_k, x.w_v, top_k=3, window=50, tokens=range(t0 + 1))
    assert torch.equal(r["out"], r2["out"])
    assert torch.equal(r["idx"], r2["idx"])


# ---------------------------------------------------------------- a7: decode

def test_decode_equals_last_prefill_row():
    B, L, hq, hkv, dk, dv = 2, 333, 4, 2, 16, 8
    d = synth.decode_inputs(B, L, hq, hkv, dk, dv, seed=6)
    seqlens = torch.tensor([L, 250], dtype=torch.int32)
    kc = oracle.compress_cache(d.k_cache, d.w_k, 32, 16)
    vc = oracle.compress_cache(d.v_cache, d.w_v, 32, 16)
    r = oracle.nsa_decode(d.q, d.k_cache, d.v_cache, kc, vc, seqlens, d.gates, top_k=3, window=40)
    for b in range(B):
        Lb = int(seqlens[b])
        q = torch.zeros(1, Lb, hq, dk, dtype=torch.bfloat16)
        q[0, Lb - 1] = d.q[b]
        gates = torch.zeros(1, Lb, hq, 3, dtype=torch.bfloat16)
        gates[0, Lb - 1] = d.gates[b]
        rp = oracle.nsa_forward(q, d.k_cache[b:b + 1, :Lb], d.v_cache[b:b + 1, :Lb], gates, d.w_k, d.w_v,
                                top_k=3, window=40, tokens=[Lb - 1])
        assert torch.allclose(r["out"][b], rp["out"][0, 0], atol=1e-13)
        assert torch.equal(r["idx"][b], rp["idx"][0, :, 0])


# ---------------------------------------------------------------- a8: MoBA

def test_moba_block_keys_are_means():
    g = torch.Generator().manual_seed(7)
    K = torch.randn(100, 3, generator=g, dtype=F64)
    kb = oracle.moba_block_keys(K, 16)
    for j in range(kb.shape[0]):
        rows = list(range(16 * j, min(100, 16 * j + 16)))
        assert torch.allclose(kb[j], sum(K[r] for r in rows) / len(rows), atol=1e-14)


def test_moba_all_blocks_is_full_causal_and_none_is_own_block():
    x = synth.moba_inputs(1, 256, 2, 8, seed=8)
    r = oracle.moba_forward(x.q, x.k, x.v, block=32, top_k=8)
    assert torch.allclose(r["out"][0], sdpa(x.q[0], x.k[0], x.v[0], causal=True), atol=1e-12)
    r0 = oracle.moba_forward(x.q, x.k, x.v, block=32, top_k=0)
    t = torch.arange(256)
    mask = (t[:, None] >= t[None, :]) & (t[:, None] // 32 == t[None, :] // 32)
    assert torch.allclose(r0["out"][0], sdpa(x.q[0], x.k[0], x.v[0], mask=mask), atol=1e-12)


def test_moba_selection_is_best_subset_per_head_and_keeps_own_block():
    x = synth.moba_inputs(1, 320, 2, 8, seed=9)
    blk, k = 32, 3
    r = oracle.moba_forward(x.q, x.k, x.v, block=blk, top_k=k)
    per_head_differs = False
    for t in range(320):
        own = t // blk
        rows = []
        for h in range(2):
            sel = [j for j in r["idx"][0, h, t].tolist() if j >= 0]
            assert sel[-1] == own and sel == sorted(sel)
            kbar = torch.stack([x.k[0, j * blk:(j + 1) * blk, h].to(F64).mean(0) for j in range(own)]) \
                if own else torch.zeros(0, 8, dtype=F64)
            sc = kbar @ x.q[0, t, h].to(F64)
            if own <= k:
                assert sel[:-1] == list(range(own))
            else:
                best = max(itertools.combinations(range(own), k), key=lambda sub: float(sc[list(sub)].sum()))
                assert sel[:-1] == sorted(best)
            rows.append(sel)
        per_head_differs |= rows[0] != rows[1]
    assert per_head_differs


# ---------------------------------------------------------------- score mappings (R3 and its alternatives)

@pytest.mark.parametrize("mapping,inside,straddle", [
    ("touch", [0, 1, 0], [1, 1, 0]),
    ("contained", [0, 1, 0], [0, 0, 0]),
    ("overlap", [0, 1, 0], [0.5, 0.5, 0]),
])
def test_score_maps_on_single_blocks(mapping, inside, straddle):
    """l = 32, s = 16, b = 64: compressed block 4 spans [64, 96), inside selection block 1;
    block 3 spans [48, 80), half in block 0 and half in block 1."""
    t = 150   # 9 visible compressed blocks, selection blocks 0..2
    p = torch.zeros(1, 9, dtype=torch.float64)
    p[0, 4] = 1.0
    assert oracle.selection_scores(p, t, 32, 16, 64, mapping).tolist() == inside
    p.zero_()
    p[0, 3] = 1.0
    assert oracle.selection_scores(p, t, 32, 16, 64, mapping).tolist() == straddle


def test_score_maps_order_and_overlap_keeps_the_mass():
    """Overlap splits each probability exactly (the scores add up to the total); contained <=
    overlap <= touch block by block; touch counts every straddling block twice."""
    g = torch.Generator().manual_seed(5)
    t = 1000
    n = oracle.num_visible_cmp_blocks(t, 32, 16, 10**6)
    p = torch.rand(4, n, generator=g, dtype=torch.float64)
    p /= p.sum(dim=1, keepdim=True)
    sc = {m: oracle.selection_scores(p, t, 32, 16, 64, m) for m in oracle.SCORE_MAPS}
    assert torch.allclose(sc["overlap"].sum(), p.sum())
    assert (sc["contained"] <= sc["overlap"] + 1e-15).all() and (sc["overlap"] <= sc["touch"] + 1e-15).all()
    straddling = p.sum(dim=0)[3::4].sum()
    assert torch.allclose(sc["touch"].sum() - sc["contained"].sum(), 2 * straddling)


def test_unknown_score_map_is_rejected():
    with pytest.raises(ValueError):
        oracle.selection_scores(torch.ones(1, 4, dtype=torch.float64), 100, 32, 16, 64, "nearest")


# ---------------------------------------------------------------- phi as a two-layer MLP (R15)

def test_gelu_matches_the_library_routine():
    x = torch.linspace(-8, 8, 1001, dtype=torch.float64)
    assert torch.allclose(oracle.gelu(x), torch.nn.functional.gelu(x), atol=1e-14, rtol=0)


def test_phi_mlp_matches_bruteforce_and_position_term_is_the_bias():
    """Block by block with explicit loops, and an intra-block position embedding added to the
    keys equals the bias vec(pe) @ W1 (the identity the library relies on)."""
    g = torch.Generator().manual_seed(7)
    T, d, l, s, h = 70, 8, 32, 16, 8
    X = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(l * d, h, generator=g, dtype=torch.float64) / 16
    W2 = torch.randn(h, d, generator=g, dtype=torch.float64) / 3
    pe = torch.randn(l, d, generator=g, dtype=torch.float64)
    b1 = pe.reshape(-1) @ W1
    got = oracle.phi_mlp(X, W1, b1, W2, l, s, round_hidden=False)
    n = (T - l) // s + 1
    assert got.shape == (n, d)
    for i in range(n):
        z = torch.zeros(h, dtype=torch.float64)
        for r in range(l):
            for c in range(d):
                z += (X[s * i + r, c] + pe[r, c]) * W1[r * d + c]
        hid = 0.5 * z * (1 + torch.erf(z / math.sqrt(2)))
        assert torch.allclose(got[i], hid @ W2, atol=1e-12, rtol=0)


def test_phi_mlp_reduces_to_the_linear_phi_in_the_linear_regime():
    """With a large bias the GELU is the identity up to exp(-b^2/2): the MLP becomes the linear
    phi with W1 @ W2 plus the constant (b1 @ W2)."""
    g = torch.Generator().manual_seed(8)
    T, d, l, s = 64, 4, 32, 16
    X = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(l * d, d, generator=g, dtype=torch.float64) / 100
    W2 = torch.randn(d, d, generator=g, dtype=torch.float64)
    b1 = torch.full((d,), 20.0, dtype=torch.float64)
    got = oracle.phi_mlp(X, W1, b1, W2, l, s, round_hidden=False)
    want = oracle.phi_compress(X, W1 @ W2, l, s) + b1 @ W2
    assert torch.allclose(got, want, atol=1e-9, rtol=0)


# ---------------------------------------------------------------- gradients (the backward's reference)

def test_oracle_gradients_match_finite_differences():
    """torch autograd through the fp64 oracle (forced block choice) against central differences
    of the same function, at a few coordinates of every input: pins that the oracle forward is
    differentiable end to end (phi, the three branches, the gates)."""
    x = synth.nsa_inputs(1, 70, 4, 1, 64, 64, seed=9)
    base = {n: getattr(x, n).double() for n in ("q", "k", "v", "gates", "w_k", "w_v")}
    first = oracle.nsa_forward(*[base[n] for n in ("q", "k", "v", "gates", "w_k", "w_v")], top_k=3, window=20,
                               round_kc=False)
    forced = first["idx"]
    g = torch.Generator().manual_seed(10)
    dout = torch.randn(first["out"].shape, generator=g, dtype=torch.float64)

    def loss(inp):
        r = oracle.nsa_forward(*[inp[n] for n in ("q", "k", "v", "gates", "w_k", "w_v")], top_k=3, window=20,
                               round_kc=False, forced_idx=forced)
        return (r["out"] * dout).sum()

    leaves = {n: t.clone().requires_grad_() for n, t in base.items()}
    loss(leaves).backward()
    for name, t in base.items():
        flat = t.reshape(-1)
        for pos in torch.randint(0, flat.numel(), (3,), generator=g).tolist():
            h = 1e-6 * max(1.0, abs(float(flat[pos])))
            up, dn = t.clone(), t.clone()
            up.reshape(-1)[pos] += h
            dn.reshape(-1)[pos] -= h
            fd = (loss({**base, name: up}) - loss({**base, name: dn})) / (2 * h)
            ad = leaves[name].grad.reshape(-1)[pos]
            assert abs(float(fd - ad)) <= 1e-5 * max(1.0, abs(float(ad))), (name, pos, float(fd), float(ad))


def test_oracle_mlp_gradients_match_finite_differences():
    """The same pin with phi as the two-layer MLP: autograd through GELU, both layers and the
    bias against central differences (hidden rows unrounded, so the function is smooth), at a
    few coordinates of every input, the MLP's weights and bias included.  The backward's MLP
    gradients (dW2 = hidden^T dXc, dpre = dXc W2^T GELU'(pre), db1 = sum of dpre) are checked
    against this autograd on the GPU."""
    x = synth.nsa_inputs(1, 70, 4, 1, 64, 64, seed=11)
    w_k, b_k, w_k2 = synth.phi_mlp_weights(32, 64, seed=12)
    w_v, b_v, w_v2 = synth.phi_mlp_weights(32, 64, seed=13)
    base = {n: t.double() for n, t in dict(q=x.q, k=x.k, v=x.v, gates=x.gates, w_k=w_k, w_v=w_v, b_k=b_k,
                                            w_k2=w_k2, b_v=b_v, w_v2=w_v2).items()}
    mlp_names = ("b_k", "w_k2", "b_v", "w_v2")
    run = lambda inp, forced=None: oracle.nsa_forward(
        *[inp[n] for n in ("q", "k", "v", "gates", "w_k", "w_v")], top_k=3, window=20, round_kc=False,
        mlp={n: inp[n] for n in mlp_names}, forced_idx=forced)
    forced = run(base)["idx"]
    g = torch.Generator().manual_seed(14)
    dout = torch.randn(run(base, forced)["out"].shape, generator=g, dtype=torch.float64)
    loss = lambda inp: (run(inp, forced)["out"] * dout).sum()
    leaves = {n: t.clone().requires_grad_() for n, t in base.items()}
    loss(leaves).backward()
    for name, t in base.items():
        flat = t.reshape(-1)
        for pos in torch.randint(0, flat.numel(), (3,), generator=g).tolist():
            h = 1e-6 * max(1.0, abs(float(flat[pos])))
            up, dn = t.clone(), t.clone()
            up.reshape(-1)[pos] += h
            dn.reshape(-1)[pos] -= h
            fd = (loss({**base, name: up}) - loss({**base, name: dn})) / (2 * h)
            ad = leaves[name].grad.reshape(-1)[pos]
            assert abs(float(fd - ad)) <= 1e-5 * max(1.0, abs(float(ad))), (name, pos, float(fd), float(ad))
