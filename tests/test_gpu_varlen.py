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
from tests.helpers import assert_close, idx_agreement, token_mask

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
        ref = oracle.nsa_forward(q[sl].unsqueeze(0), k[sl].unsqueeze(0), v[sl].unsqueeze(0),
                                 gates[sl].unsqueeze(0), w_k, w_v, top_k=top_k, window=window)
        toks = ref["tokens"]
        gi = idx[b:b + 1, :, toks]
        _, swapped = idx_agreement(gi, ref["idx"], ref["score"], tokens=toks)
        mask = token_mask((1, len(toks), hq), swapped, hq // hkv)
        assert_close(out[sl].unsqueeze(0)[:, toks], ref["out"],
                     mask=mask.unsqueeze(-1).expand(-1, -1, -1, dv), what=f"out of sequence {b}")
