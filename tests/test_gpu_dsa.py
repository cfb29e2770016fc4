"""GPU parity of the DSA forward (nsa_dsa_forward: lightning indexer, token-wise top-k,
attention over the chosen tokens) against the fp64 oracle on the same seeded inputs."""
import dataclasses

import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from tests.helpers import assert_close, check_swap, with_forced_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
NEAR_TIE = 1e-4   # relative: a chosen token may differ from the oracle's only within this of the k-th score


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def run_gpu(x, top_k):
    B, T, hq, dk = x.q.shape
    hkv, dv = x.k.shape[2], x.v.shape[3]
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.q_idx, x.k_idx, x.w_idx)]
    cfg = nsa.make_config(mode=nsa.NSA_MODE_DSA, batch=B, seqlen=T, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=top_k)
    ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.empty((B, T, hq, dv), dtype=torch.bfloat16, device=DEV)
    sel = torch.full((B, T, top_k), -7, dtype=torch.int32, device=DEV)
    nsa.nsa_dsa_forward(*dev, cfg, out, sel_out=sel)
    torch.cuda.synchronize()
    return out.cpu(), sel.cpu()


def check(x, top_k, tokens, min_exact=0.97, out_sel=None):
    """Chosen tokens: ascending, causal, distinct, and bit-exact except legal near-tie swaps
    (check_swap with a tie width relative to the k-th score).  Every output row is compared,
    those with a swap against the oracle in forced-index mode on the GPU's choice."""
    out, sel = run_gpu(x, top_k) if out_sel is None else out_sel
    run = lambda toks, forced=None: oracle.dsa_forward(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w_idx, top_k=top_k,
                                                       tokens=toks, forced_idx=forced)
    ref = run(tokens)
    B = x.q.shape[0]
    exact = 0
    swapped = set()
    for b in range(B):
        for n, t in enumerate(tokens):
            a = sel[b, t].tolist()
            o = ref["idx"][b, n].tolist()
            m = min(t + 1, top_k)
            assert a[:m] == sorted(a[:m]) and all(0 <= j <= t for j in a[:m]) and a[m:] == [-1] * (top_k - m), (b, t)
            if a == o:
                exact += 1
                continue
            sc = ref["score"][b][n]
            kth = sorted(sc.tolist(), reverse=True)[m - 1]
            check_swap(a[:m], o[:m], sc, (), NEAR_TIE * max(1.0, abs(kth)), (b, t))
            swapped.add((b, n))
    assert exact >= min_exact * B * len(tokens), exact
    ref_out = with_forced_rows(ref["out"], swapped,
                               lambda pos: run([tokens[i] for i in pos], sel[:, [tokens[i] for i in pos]])["out"])
    assert_close(out[:, tokens], ref_out, what="dsa out")
    return len(swapped)


def test_dsa_group_of_16():
    x = synth.dsa_inputs(1, 700, 32, 2, 192, 128, 4, 64, seed=71)
    check(x, 64, tokens=[0, 1, 5, 63, 64, 65, 200, 411, 699])


def test_dsa_small_heads_and_batch():
    x = synth.dsa_inputs(2, 333, 4, 1, 64, 64, 2, 128, seed=72)
    check(x, 16, tokens=list(range(0, 333, 7)))


def test_dsa_every_token_chosen_is_full_causal_attention():
    """top_k >= T: the indexer no longer matters; the output is full causal attention."""
    x = synth.dsa_inputs(1, 130, 16, 1, 128, 128, 3, 64, seed=73)
    check(x, 256, tokens=list(range(130)), min_exact=1.0)


def test_dsa_benchmark_workload_sampled():
    """The workload the benchmark times: T = 8192, 64 query heads in 4 groups, d_k 192,
    d_v 128, 4 indexer heads of 64 dims, top-2048 (the radix select's large-k path and the
    full [T, T] score matrix); sampled tokens against the oracle."""
    c = synth.WORKLOADS["dsa_8k"]
    x = synth.dsa_inputs(c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"], c["h_i"], c["d_i"], seed=0)
    g = torch.Generator().manual_seed(74)
    T = c["T"]
    toks = sorted(set([0, 1, 2046, 2047, 2048, 2049, 4095, T - 1] + torch.randint(0, T, (24,), generator=g).tolist()))
    check(x, c["top_k"], toks)


@pytest.mark.parametrize("hi,di", [(24, 64), (12, 128)])
def test_dsa_many_indexer_heads(hi, di):
    """More indexer heads than the select kernel keeps in shared memory: the query fragments
    come from global memory per head and tile (the other code path of the score tile)."""
    x = synth.dsa_inputs(1, 600, 16, 1, 128, 128, hi, di, seed=75)
    check(x, 96, tokens=[0, 95, 96, 97, 300, 511, 599])


def test_dsa_exact_ties_take_the_lowest_indices():
    """Indexer keys repeating every 5 tokens give each query only 5 distinct scores, each held
    by ~T/5 tokens, so the k-th score is shared by many: the choice must be the lowest indices
    among the equal ones, exactly as the oracle takes them (scores equal bit for bit on both
    sides, since the rows are equal)."""
    x = synth.dsa_inputs(1, 900, 16, 1, 128, 128, 2, 64, seed=76)
    k_idx = x.k_idx.clone()
    k_idx[0] = k_idx[0, torch.arange(900) % 5]
    x = dataclasses.replace(x, k_idx=k_idx)
    check(x, 100, tokens=[99, 100, 101, 250, 513, 640, 899], min_exact=1.0)


def test_dsa_zero_weights_take_the_first_tokens():
    """A token whose indexer weights are all zero scores every earlier token 0: it takes the
    first top_k tokens."""
    x = synth.dsa_inputs(1, 500, 16, 1, 128, 128, 4, 64, seed=77)
    w = x.w_idx.clone()
    w[0, 300] = 0
    w[0, 450] = 0
    x = dataclasses.replace(x, w_idx=w)
    out, sel = run_gpu(x, 64)
    assert sel[0, 300].tolist() == list(range(64)) and sel[0, 450].tolist() == list(range(64))
    check(x, 64, tokens=[300, 450, 499], out_sel=(out, sel), min_exact=1.0)


def test_dsa_32k_runs_with_workspace_of_the_chosen_tokens_only():
    """T = 32768 with top-2048: the workspace holds only the status word and the chosen tokens
    (O(T * top_k), no [T, T] score matrix); sampled tokens against the oracle."""
    T, K = 32768, 2048
    x = synth.dsa_inputs(1, T, 16, 1, 128, 128, 4, 64, seed=78)
    cfg = nsa.make_config(mode=nsa.NSA_MODE_DSA, batch=1, seqlen=T, h_q=16, h_kv=1, d_k=128, d_v=128, top_k=K)
    up = lambda n: (n + 255) // 256 * 256
    assert nsa.nsa_workspace_size(cfg) == 256 + up(T * K * 4)
    g = torch.Generator().manual_seed(79)
    toks = sorted(set([0, K - 1, K, T - 1] + torch.randint(K, T, (12,), generator=g).tolist()))
    check(x, K, toks)
