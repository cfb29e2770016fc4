"""Comparison rules shared by the GPU parity tests (tests only)."""
from __future__ import annotations

import torch

MAX_ABS = 2e-2      # output tolerance for bf16 inputs with fp32 accumulation
MEAN_ABS = 2e-3
NEAR_TIE = 1e-3     # index choices may differ only where the oracle's score gap is below this


def idx_agreement(gpu_idx, ora_idx, scores, forced=(True, True), sel_block=64, tokens=None):
    """Compare chosen blocks per (b, g, n).  Returns (n_exact, swapped_set); raises
    AssertionError on any choice that is not a legal near-tie swap.

    gpu_idx, ora_idx: [B, G, n, k] int tensors (n = len(tokens)); scores[b][g][n] is
    the oracle's score vector of that token."""
    gpu_idx = gpu_idx.cpu().long()
    ora_idx = ora_idx.cpu().long()
    B, G, n, k = ora_idx.shape
    swapped = set()
    exact = 0
    for b in range(B):
        for g in range(G):
            for i in range(n):
                a = gpu_idx[b, g, i].tolist()
                o = ora_idx[b, g, i].tolist()
                if a == o:
                    exact += 1
                    continue
                t = tokens[i] if tokens is not None else i
                sc = scores[b][g][i]
                forced_set = set()
                if forced[0]:
                    forced_set.add(0)
                if forced[1]:
                    forced_set.add(t // sel_block)
                so, sa = set(j for j in o if j >= 0), set(j for j in a if j >= 0)
                assert len(sa) == len(so), (b, g, t, a, o)
                assert a == sorted(a[:len(sa)]) + [-1] * (k - len(sa)), (b, g, t, a)
                assert forced_set <= sa, (b, g, t, a)
                free = [j for j in so if j not in forced_set]
                thr = min(float(sc[j]) for j in free)
                for j in sa - so:
                    assert 0 <= j <= t // sel_block, (b, g, t, a)
                    assert float(sc[j]) >= thr - NEAR_TIE, (b, g, t, j, float(sc[j]), thr)
                swapped.add((b, g, i))
    return exact, swapped


def assert_close(gpu, ref, mask=None, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    d = (gpu.detach().cpu().double() - ref.double()).abs()
    if mask is not None:
        d = d[mask]
    assert d.numel() > 0, what
    mx, mn = float(d.max()), float(d.mean())
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max {mx:.3e} mean {mn:.3e}"
    return mx, mn


def token_mask(shape_bn_h, swapped, G):
    """Mask [B, n, H] that drops the heads of (b, g, n) entries whose choice was a near-tie swap."""
    B, n, H = shape_bn_h
    m = torch.ones((B, n, H), dtype=torch.bool)
    for (b, g, i) in swapped:
        m[b, i, g * G:(g + 1) * G] = False
    return m


def assert_phi_close(got, x, w, what="phi"):
    """GPU phi (fp32 accumulation, one bf16 rounding) against the exact fp64 map:
    |got - exact| <= 2^-8 |exact| (the rounding) + 2^-17 * (|x| @ |w|) (fp32 accumulation
    over l*d terms).  Also most entries round to exactly the same bf16 value."""
    import oracle
    exact = oracle.compress_cache(x, w, 32, 16, round_kc=False)
    mag = oracle.compress_cache(x.double().abs(), w.double().abs(), 32, 16, round_kc=False)
    got = got.detach().cpu().double()
    assert got.shape == exact.shape, what
    if exact.numel() == 0:
        return
    bad = (got - exact).abs() > exact.abs() * 2 ** -8 + mag * 2 ** -17
    assert not bad.any(), f"{what}: {int(bad.sum())} entries off"
    differ = int((got != oracle.round_bf16(exact)).sum())
    assert differ <= max(8, exact.numel() // 100), f"{what}: {differ} of {exact.numel()} differ after rounding"
