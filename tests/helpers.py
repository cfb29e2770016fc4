"""Comparison rules shared by the GPU parity tests (tests only).

Block choices: where the oracle's scores leave a near tie at the top-k boundary, more
than one choice is correct.  A GPU choice that differs from the oracle's must then be a
legal near-tie swap: every block it added scores at least the lowest free block the
oracle chose minus the tie width, and every block it dropped scores at most the lowest
free block it kept plus the tie width (so no clearly better block was left out).
Outputs: every compared row is checked.  The rows whose choice is a legal swap are
compared with the oracle run in forced-index mode on the GPU's choice, the rows with the
oracle's own choice with the oracle's output.
"""
from __future__ import annotations

import torch

MAX_ABS = 2e-2      # output tolerance for bf16 inputs with fp32 accumulation
MEAN_ABS = 2e-3
NEAR_TIE = 1e-3     # index choices may differ only where the oracle's score gap is below this


def check_swap(gpu_sel, ora_sel, score, fixed, eps, where=()):
    """Assert that the set gpu_sel (ints) is a legal near-tie variant of ora_sel under the
    oracle's ``score`` (indexable by block); ``fixed`` are the blocks both must hold."""
    sa, so = set(gpu_sel), set(ora_sel)
    assert len(sa) == len(gpu_sel) and len(sa) == len(so), (where, gpu_sel, ora_sel)
    assert set(fixed) <= sa and set(fixed) <= so, (where, gpu_sel, fixed)
    added, dropped = sa - so, so - sa
    if not added:
        return
    ora_free = [j for j in so if j not in fixed]
    gpu_free = [j for j in sa if j not in fixed]
    thr_o = min(float(score[j]) for j in ora_free)
    thr_g = min(float(score[j]) for j in gpu_free)
    for j in added:
        assert float(score[j]) >= thr_o - eps, ("added", where, j, float(score[j]), thr_o)
    for j in dropped:
        assert float(score[j]) <= thr_g + eps, ("dropped", where, j, float(score[j]), thr_g)


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
                forced_set = set()
                if forced[0]:
                    forced_set.add(0)
                if forced[1]:
                    forced_set.add(t // sel_block)
                sa = [j for j in a if j >= 0]
                assert a == sorted(sa) + [-1] * (k - len(sa)), (b, g, t, a)
                assert all(0 <= j <= t // sel_block for j in sa), (b, g, t, a)
                check_swap(sa, [j for j in o if j >= 0], scores[b][g][i], forced_set, NEAR_TIE, (b, g, t))
                swapped.add((b, g, i))
    return exact, swapped


def swapped_tokens(swapped):
    """Sorted positions i (in the compared token list) of the entries with a legal swap."""
    return sorted(set(e[-1] for e in swapped))


def with_forced_rows(ref_out, swapped, rerun):
    """ref_out [B, n, ...] with the rows of every swapped token position replaced by
    rerun(positions) (the oracle in forced-index mode on the GPU's choice, [B, m, ...])."""
    pos = swapped_tokens(swapped)
    if not pos:
        return ref_out
    out = ref_out.clone()
    out[:, pos] = rerun(pos)
    return out


def assert_close(gpu, ref, mask=None, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    d = (gpu.detach().cpu().double() - ref.double()).abs()
    if mask is not None:
        d = d[mask]
    assert d.numel() > 0, what
    mx, mn = float(d.max()), float(d.mean())
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max {mx:.3e} mean {mn:.3e}"
    return mx, mn


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
