"""GPU parity of the MoBA mode of nsa_forward (through the C ABI) against the
fp64 CPU oracle on the same seeded inputs."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from tests.helpers import NEAR_TIE, assert_close, check_swap

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def run_moba(x, block, top_k):
    B, T, H, d = x.q.shape
    q, k, v = (t.to(DEV) for t in (x.q, x.k, x.v))
    idx = torch.full((B, H, T, top_k + 1), -7, dtype=torch.int32, device=DEV)
    out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=DEV)
    cfg = nsa.make_config(mode=nsa.NSA_MODE_MOBA, batch=B, seqlen=T, h_q=H, h_kv=H, d_k=d, d_v=d, sel_block=block,
                          top_k=top_k, w_cmp_k=None, w_cmp_v=None, sel_idx_out=idx)
    ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    nsa.nsa_forward(q, k, v, None, cfg, out)
    torch.cuda.synchronize()
    return out.cpu(), idx.cpu()


def compare(out, idx, ref, heads, rerun, min_exact=0.98):
    """Choices bit-exact except legal near-tie swaps (check_swap: the own block kept last, each
    added past block within NEAR_TIE of the oracle's lowest pick, each dropped one within
    NEAR_TIE of the GPU's lowest pick); every output row compared, the swapped (token, head)
    rows against the oracle in forced-index mode on the GPU's choice (``rerun(tokens, forced)``
    with forced [B, H, n, top_k+1] returns the oracle's output [B, n, H, d])."""
    B, n, H, d = ref["out"].shape
    toks = ref["tokens"]
    exact = total = 0
    swapped = set()
    for b in range(B):
        for hi, h in enumerate(heads):
            for i, t in enumerate(toks):
                g = idx[b, h, t].tolist()
                o = ref["idx"][b, h, i].tolist()
                total += 1
                if g == o:
                    exact += 1
                    continue
                sg, so = [j for j in g if j >= 0], [j for j in o if j >= 0]
                own = t // ref["block"]
                assert sg[-1] == own and so[-1] == own, (b, h, t, g, o)
                assert sg[:-1] == sorted(sg[:-1]) and all(0 <= j < own for j in sg[:-1]), (b, h, t, g)
                check_swap(sg[:-1], so[:-1], ref["score"][(b, h, i)], (), NEAR_TIE, (b, h, t))
                swapped.add((b, hi, i))
    assert exact >= min_exact * total, (exact, total)
    ref_out = ref["out"].clone()
    pos = sorted(set(i for (_, _, i) in swapped))
    if pos:
        forced = idx[:, :, [toks[i] for i in pos]].long()
        ref_out[:, pos] = rerun([toks[i] for i in pos], forced)
    return assert_close(out[:, toks][:, :, list(heads)], ref_out, what="moba out")


@pytest.mark.parametrize("T,H,block,top_k", [(2048, 4, 256, 3), (1000, 2, 64, 2), (640, 2, 64, 5)])
def test_moba_full(T, H, block, top_k):
    x = synth.moba_inputs(1, T, H, 128, seed=31)
    out, idx = run_moba(x, block, top_k)
    run = lambda toks, forced=None: oracle.moba_forward(x.q, x.k, x.v, block=block, top_k=top_k, tokens=toks,
                                                        forced_idx=forced)
    ref = run(None)
    ref["block"] = block
    compare(out, idx, ref, range(H), lambda toks, forced: run(toks, forced)["out"])


def test_moba_no_past_block_is_block_local_attention():
    T, H, block = 700, 2, 128
    x = synth.moba_inputs(1, T, H, 128, seed=32)
    out, idx = run_moba(x, block, 0)
    t = torch.arange(T)
    mask = (t[:, None] >= t[None, :]) & (t[:, None] // block == t[None, :] // block)
    q, k, v = (a[0].double().transpose(0, 1) for a in (x.q, x.k, x.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask).transpose(0, 1)
    assert_close(out[0], ref, what="block-local")
    assert (idx[0, :, :, 0] == (t // block).to(torch.int32)).all()


def test_moba_every_block_is_full_causal():
    T, H = 768, 2
    x = synth.moba_inputs(1, T, H, 128, seed=33)
    out, _ = run_moba(x, 256, 2)      # 3 blocks of 256: every past block is chosen
    q, k, v = (a[0].double().transpose(0, 1) for a in (x.q, x.k, x.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(0, 1)
    assert_close(out[0], ref, what="full causal")


def test_moba_workload_sampled():
    """The 128K-token, 32-head workload in the benchmark's launch configuration;
    sampled tokens of four heads are checked against the oracle."""
    c = synth.WORKLOADS["moba_128k"]
    x = synth.moba_inputs(1, c["T"], c["h"], c["d"], seed=0)
    out, idx = run_moba(x, c["block"], c["top_k"])
    g = torch.Generator().manual_seed(5)
    toks = sorted(set([0, 511, 512, 1535, 1536, c["T"] - 1] + torch.randint(0, c["T"], (40,), generator=g).tolist()))
    heads = [0, 7, 19, 31]

    def run(toks_, forced=None):
        # the oracle on the checked heads only (q/k/v sliced to them; forced choices come sliced)
        sub = lambda a: a[:, :, heads]
        return oracle.moba_forward(sub(x.q), sub(x.k), sub(x.v), block=c["block"], top_k=c["top_k"], tokens=toks_,
                                   forced_idx=forced)
    ref = run(toks)
    ref["block"] = c["block"]
    sub_idx = idx[:, heads]
    compare(out[:, :, heads], sub_idx, ref, range(len(heads)), lambda t_, f_: run(t_, f_)["out"], min_exact=0.95)
