"""GPU tests of the variable-length prefill (nsa_forward_varlen): a packed batch of
sequences of different lengths, each computed as if alone.

- Every output row and every chosen block equals, bit for bit, what nsa_forward computes for
  that sequence alone (the same kernels take the same decisions on the same rows).
- A small packed batch also matches the fp64 oracle run per sequence.
"""
import pytest
import torch

import oracle
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward, NSAForwardVarlen
from tests.helpers import assert_close, idx_agreement, with_forced_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def packed_inputs(lengths, hq, hkv, dk, dv, seed):
    x, cu = synth.nsa_varlen_inputs(lengths, hq, hkv, dk, dv, seed=seed)
    return x.q, x.k, x.v, x.gates, x.w_k, x.w_v, cu


def run_varlen(lengths, hq, hkv, dk, dv, top_k, window, seed):
    q, k, v, gates, w_k, w_v, cu = packed_inputs(lengths, hq, hkv, dk, dv, seed)
    T = max(lengths)
    dev = [t.to(DEV) for t in (q, k, v, gates, w_k, w_v, cu)]
    f = NSAForwardVarlen(len(lengths), T, hq, hkv, dk, dv, dev[4], dev[5], top_k=top_k, window=window)
    out = f(*dev[:4], dev[6])
    torch.cuda.synchronize()
    assert f.device_status() == 0
    return (q, k, v, gates, w_k, w_v, cu), out.cpu(), f.idx.cpu(), f.kc.cpu(), f.vc.cpu()


@pytest.mark.parametrize("lengths,dk", [
    ([700, 1, 33, 0, 1300, 64, 129, 8], 192),   # ragged, empty, shorter than a compression block
    ([517, 2048, 95], 128),
])
def test_varlen_equals_each_sequence_alone(lengths, dk):
    hq, hkv, dv, top_k, window = 32, 2, 128, 16, 512
    (q, k, v, gates, w_k, w_v, cu), out, idx, kc, vc = run_varlen(lengths, hq, hkv, dk, dv, top_k, window, seed=40)
    wk, wv = w_k.to(DEV), w_v.to(DEV)
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        lo = int(cu[b])
        f = NSAForward(1, L, hq, hkv, dk, dv, wk, wv, top_k=top_k, window=window)
        ref = f(q[lo:lo + L].unsqueeze(0).to(DEV), k[lo:lo + L].unsqueeze(0).to(DEV),
                v[lo:lo + L].unsqueeze(0).to(DEV), gates[lo:lo + L].unsqueeze(0).to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(out[lo:lo + L], ref[0].cpu()), f"sequence {b} (length {L}): output differs"
        assert torch.equal(idx[b, :, :L], f.idx[0].cpu()), f"sequence {b}: chosen blocks differ"
        nc = f.kc.shape[1]
        assert torch.equal(kc[b, :nc], f.kc[0].cpu()) and torch.equal(vc[b, :nc], f.vc[0].cpu())
        assert not kc[b, nc:].any() and not vc[b, nc:].any(), "rows past the sequence's blocks are zero"


def test_varlen_matches_oracle_per_sequence():
    lengths = [300, 37, 129]
    hq, hkv, dk, dv, top_k, window = 16, 1, 192, 128, 4, 100
    (q, k, v, gates, w_k, w_v, cu), out, idx, _, _ = run_varlen(lengths, hq, hkv, dk, dv, top_k, window, seed=50)
    for b, L in enumerate(lengths):
        lo = int(cu[b])
        sl = slice(lo, lo + L)
        check_sequence_against_oracle(q[sl], k[sl], v[sl], gates[sl], w_k, w_v, out[sl], idx[b, :, :L], top_k,
                                      window, None, f"sequence {b}")


def check_sequence_against_oracle(q, k, v, gates, w_k, w_v, out, idx, top_k, window, tokens, what):
    """One sequence of a packed batch (rows [L, ...], chosen blocks [H_kv, L, k]) against the
    oracle run on that sequence alone, at ``tokens`` (all if None)."""
    run_oracle = lambda toks_, forced=None: oracle.nsa_forward(
        q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), gates.unsqueeze(0), w_k, w_v, top_k=top_k, window=window,
        tokens=toks_, forced_idx=forced)
    ref = run_oracle(tokens)
    toks = ref["tokens"]
    gi = idx.unsqueeze(0)[:, :, toks]
    exact, swapped = idx_agreement(gi, ref["idx"], ref["score"], tokens=toks)
    assert exact >= 0.97 * gi.shape[1] * gi.shape[2], what
    ref_out = with_forced_rows(ref["out"], swapped,
                               lambda pos: run_oracle([toks[i] for i in pos], gi[:, :, pos])["out"])
    assert_close(out.unsqueeze(0)[:, toks], ref_out, what=f"out of {what}")


def test_varlen_benchmark_batch():
    """The packed batch the benchmark times (8 sequences, 65,536 tokens, the longest 16,384):
    each sequence bit-equal to nsa_forward on it alone, and sampled tokens of the longest and
    the shortest sequence against the oracle."""
    import synth as _s
    c = _s.WORKLOADS["nsa_varlen"]
    lengths = list(c["lengths"])
    hq, hkv, dk, dv, top_k, window = c["h_q"], c["h_kv"], c["d_k"], c["d_v"], c["top_k"], c["window"]
    (q, k, v, gates, w_k, w_v, cu), out, idx, _, _ = run_varlen(lengths, hq, hkv, dk, dv, top_k, window, seed=0)
    wk, wv = w_k.to(DEV), w_v.to(DEV)
    for b, L in enumerate(lengths):
        lo = int(cu[b])
        f = NSAForward(1, L, hq, hkv, dk, dv, wk, wv, top_k=top_k, window=window)
        ref = f(q[lo:lo + L].unsqueeze(0).to(DEV), k[lo:lo + L].unsqueeze(0).to(DEV),
                v[lo:lo + L].unsqueeze(0).to(DEV), gates[lo:lo + L].unsqueeze(0).to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(out[lo:lo + L], ref[0].cpu()), f"sequence {b} (length {L}): output differs"
        assert torch.equal(idx[b, :, :L], f.idx[0].cpu()), f"sequence {b}: chosen blocks differ"
        del f, ref
    g = torch.Generator().manual_seed(41)
    for b in (0, len(lengths) - 1):
        L, lo = lengths[b], int(cu[b])
        toks = sorted(set([0, 63, 64, 511, 512, L // 2, L - 1] + torch.randint(0, L, (24,), generator=g).tolist()))
        sl = slice(lo, lo + L)
        check_sequence_against_oracle(q[sl], k[sl], v[sl], gates[sl], w_k, w_v, out[sl], idx[b, :, :L], top_k,
                                      window, toks, f"sequence {b} (length {L})")


def clamped_ranges(cu, T, total):
    """The checked copy of cu_seqlens the library's kernels read (include/nsa.h,
    nsa_forward_varlen): each length clamped to [0, T], the running sum stopped at total."""
    safe, run = [0], 0
    for b in range(len(cu) - 1):
        run = min(run + min(max(cu[b + 1] - cu[b], 0), T), total)
        safe.append(run)
    return safe


@pytest.mark.parametrize("bad", [
    [0, 400, 437, 466],   # a length above T
    [0, 300, 200, 466],   # decreasing
    [0, 100, 200, 900],   # cu[B] past the packed rows
    [50, 100, 200, 300],  # cu[0] != 0
    [0, -5, 100, 466],    # negative
])
def test_varlen_cu_seqlens_outside_its_rules(bad):
    """Contents of cu_seqlens that break its rules are reported by the status word
    (NSA_CODE_CU_SEQLENS, nsa_device_status -> NSA_ERR_INVALID_ARG), and the kernels ran on the
    clamped ranges: the output equals, bit for bit, a call made with those ranges."""
    import block_sparse_attention_compress_b200 as nsa
    lengths = [300, 37, 129]
    hq, hkv, dk, dv, top_k, window = 16, 1, 192, 128, 4, 100
    q, k, v, gates, w_k, w_v, _ = packed_inputs(lengths, hq, hkv, dk, dv, seed=52)
    total, T = q.shape[0], max(lengths)
    safe = clamped_ranges(bad, T, total)
    assert safe != bad or bad[-1] != total
    dq, dkk, dvv, dg, wk, wv = (t.to(DEV) for t in (q, k, v, gates, w_k, w_v))
    f = NSAForwardVarlen(len(lengths), T, hq, hkv, dk, dv, wk, wv, top_k=top_k, window=window)
    out = f(dq, dkk, dvv, dg, torch.tensor(bad, dtype=torch.int32, device=DEV))
    st, word = nsa.nsa_device_status(f.workspace)
    assert (st, word) == (nsa.NSA_ERR_INVALID_ARG, nsa.NSA_CODE_CU_SEQLENS)
    n = safe[-1]
    ref_f = NSAForwardVarlen(len(lengths), T, hq, hkv, dk, dv, wk, wv, top_k=top_k, window=window)
    ref = ref_f(dq[:n], dkk[:n], dvv[:n], dg[:n], torch.tensor(safe, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert ref_f.device_status() == 0, "the clamped ranges keep every rule"
    assert torch.equal(out[:n].cpu(), ref.cpu())
    for b in range(len(lengths)):
        L = safe[b + 1] - safe[b]
        assert torch.equal(f.idx[b, :, :L].cpu(), ref_f.idx[b, :, :L].cpu()), f"sequence {b}: chosen blocks"
