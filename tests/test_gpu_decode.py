"""GPU parity of nsa_decode (one new token per sequence, through the C ABI)
against the fp64 CPU oracle on the same seeded caches."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward, compress_torch
from tests.helpers import assert_close, idx_agreement

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def run_decode(d, seqlens, top_k, window, Lmax=None, score_map=0):
    B, L, hkv, dk = d.k_cache.shape
    hq, dv = d.q.shape[1], d.v_cache.shape[3]
    dev = lambda t: t.to(DEV)
    k, v = dev(d.k_cache), dev(d.v_cache)
    kc, vc = compress_torch(k, dev(d.w_k)), compress_torch(v, dev(d.w_v))
    idx = torch.full((B, hkv, top_k), -7, dtype=torch.int32, device=DEV)
    out = torch.empty((B, hq, dv), dtype=torch.bfloat16, device=DEV)
    cfg = nsa.make_config(batch=B, seqlen=L, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=top_k, window=window,
                          w_cmp_k=d.w_k, w_cmp_v=d.w_v, sel_idx_out=idx, score_map=score_map)
    ws = torch.empty(max(nsa.nsa_workspace_size(cfg, B), 4), dtype=torch.uint8, device=DEV)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    sl = dev(seqlens.to(torch.int32))
    nsa.nsa_decode(dev(d.q), k, v, kc, vc, sl, int(seqlens.max()), dev(d.gates), cfg, out)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a device-side wait timed out"
    return out.cpu(), idx.cpu()


def check(d, seqlens, top_k, window, batch=None, score_map=0):
    """Every sequence's output against the oracle: where the GPU's block choice for a group
    differs from the oracle's by a legal near-tie swap, the oracle reruns that sequence on the
    GPU's blocks (forced-index mode) and that group's rows are compared with the rerun."""
    out, idx = run_decode(d, seqlens, top_k, window, score_map=score_map)
    bs = list(range(d.q.shape[0])) if batch is None else batch
    sub = lambda t: t[bs]
    kc = oracle.compress_cache(sub(d.k_cache), d.w_k, 32, 16)
    vc = oracle.compress_cache(sub(d.v_cache), d.w_v, 32, 16)
    run = lambda rows, forced=None: oracle.nsa_decode(
        sub(d.q), sub(d.k_cache), sub(d.v_cache), kc, vc, seqlens[bs], sub(d.gates), top_k=top_k, window=window,
        score_map=oracle.SCORE_MAPS[score_map], batch=rows, forced_idx=forced)
    ref = run(None)
    toks = [int(seqlens[b]) - 1 for b in bs]
    gi = idx[bs]
    hq, hkv = d.q.shape[1], d.k_cache.shape[2]
    G = hq // hkv
    n_exact = 0
    ref_out = ref["out"].clone()
    for i in range(len(bs)):
        swapped_groups = []
        for g in range(hkv):
            e, sw = idx_agreement(gi[i:i + 1, g:g + 1].unsqueeze(2), ref["idx"][i:i + 1, g:g + 1].unsqueeze(2),
                                  [[[ref["score"][i][g]]]], tokens=[toks[i]])
            n_exact += e
            if sw:
                swapped_groups.append(g)
        if swapped_groups:
            forced = run([i], gi[i:i + 1])["out"][0]
            for g in swapped_groups:
                ref_out[i, g * G:(g + 1) * G] = forced[g * G:(g + 1) * G]
    assert n_exact >= 0.9 * len(bs) * hkv
    assert_close(out[bs], ref_out, what="decode out")
    return n_exact


def test_decode_varlen_small():
    B, L = 6, 3000
    d = synth.decode_inputs(B, L, 64, 4, 192, 128, seed=21)
    seqlens = torch.tensor([3000, 1, 31, 32, 777, 2049], dtype=torch.int32)
    check(d, seqlens, 16, 512)


def test_decode_tiny_heads():
    d = synth.decode_inputs(2, 1024, 4, 1, 64, 64, seed=22)
    check(d, torch.tensor([1024, 600], dtype=torch.int32), 4, 128)


def test_decode_head_dim_128():
    d = synth.decode_inputs(3, 2600, 32, 2, 128, 128, seed=24)
    check(d, torch.tensor([2600, 65, 1999], dtype=torch.int32), 16, 256)


def test_decode_matches_last_prefill_row_on_gpu():
    """The decode step at position L-1 and the prefill's last row are the same arithmetic."""
    L = 1500
    x = synth.nsa_inputs(1, L, 64, 4, 192, 128, seed=23)
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.gates, x.w_k, x.w_v)]
    f = NSAForward(1, L, 64, 4, 192, 128, dev[4], dev[5], top_k=16, window=512)
    pre = f(*dev[:4])
    d = synth.DecodeInputs(q=x.q[:, L - 1], k_cache=x.k, v_cache=x.v, w_k=x.w_k, w_v=x.w_v,
                           gates=x.gates[:, L - 1], seqlens=torch.tensor([L], dtype=torch.int32))
    out, idx = run_decode(d, d.seqlens, 16, 512)
    assert torch.equal(idx[0], f.idx[0, :, L - 1].cpu())
    assert_close(out[0], pre[0, L - 1].cpu().double(), max_abs=1e-2, mean_abs=1e-3, what="decode vs prefill")


def test_decode_workload_sampled():
    """The 32 x 65536 decode workload in the benchmark's launch configuration; three
    sequences are checked against the oracle."""
    c = synth.WORKLOADS["nsa_decode"]
    d = synth.decode_inputs(c["B"], c["L"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"], seed=0, device=DEV)
    out, idx = run_decode(d, d.seqlens.cpu(), c["top_k"], c["window"])
    host = synth.DecodeInputs(*(t.cpu() for t in (d.q, d.k_cache, d.v_cache, d.w_k, d.w_v, d.gates, d.seqlens)))
    del d
    torch.cuda.empty_cache()
    bs = [0, 13, 31]
    sub = lambda t: t[bs]
    kc = oracle.compress_cache(sub(host.k_cache), host.w_k, 32, 16)
    vc = oracle.compress_cache(sub(host.v_cache), host.w_v, 32, 16)
    run = lambda rows, forced=None: oracle.nsa_decode(
        sub(host.q), sub(host.k_cache), sub(host.v_cache), kc, vc, host.seqlens[bs], sub(host.gates),
        top_k=c["top_k"], window=c["window"], batch=rows, forced_idx=forced)
    ref = run(None)
    G = c["h_q"] // c["h_kv"]
    ref_out = ref["out"].clone()
    for i, b in enumerate(bs):
        swapped_groups = []
        for g in range(c["h_kv"]):
            _, sw = idx_agreement(idx[b:b + 1, g:g + 1].unsqueeze(2), ref["idx"][i:i + 1, g:g + 1].unsqueeze(2),
                                  [[[ref["score"][i][g]]]], tokens=[c["L"] - 1])
            if sw:
                swapped_groups.append(g)
        if swapped_groups:   # the oracle on the GPU's blocks for this sequence
            forced = run([i], idx[b:b + 1])["out"][0]
            for g in swapped_groups:
                ref_out[i, g * G:(g + 1) * G] = forced[g * G:(g + 1) * G]
    assert_close(out[bs], ref_out, what="decode 64K")


@pytest.mark.parametrize("score_map", [1, 2])
def test_decode_score_maps(score_map):
    """The contained and overlap readings of the compressed-to-selection mapping in decode."""
    d = synth.decode_inputs(4, 2100, 64, 4, 192, 128, seed=63)
    check(d, torch.tensor([2100, 1500, 95, 1025], dtype=torch.int32), 16, 512, score_map=score_map)
