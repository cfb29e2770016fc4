"""nsa_forward_noalloc, the entry point for callers that cannot allocate device
memory (for instance a plugin whose host application owns every allocation):
through the C ABI its output and chosen blocks must match nsa_forward, the entry
point that takes a caller-allocated workspace, on two calls in a row with
different problems sharing the same built-in scratch array.

This file is named so that pytest collects it last."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import n_cmp
from tests.helpers import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    nsa.load_library()


def _problem(B, T, hq, hkv, dk, dv, top_k, window, seed):
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=seed, device="cpu")
    d = {n: getattr(x, n).to(DEV) for n in ("q", "k", "v", "gates", "w_k", "w_v")}
    return d, dict(batch=B, seqlen=T, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=top_k, window=window)


def _run_both(d, shape):
    B, T, hq, hkv, dk, dv = (shape[k] for k in ("batch", "seqlen", "h_q", "h_kv", "d_k", "d_v"))
    outs, idxs = [], []
    for noalloc in (False, True):
        idx = torch.full((B, hkv, T, shape["top_k"]), -7, dtype=torch.int32, device=DEV)
        out = torch.full((B, T, hq, dv), float("nan"), dtype=torch.bfloat16, device=DEV)
        cfg = nsa.make_config(w_cmp_k=d["w_k"], w_cmp_v=d["w_v"], sel_idx_out=idx, **shape)
        if noalloc:
            nsa.nsa_forward_noalloc(d["q"], d["k"], d["v"], d["gates"], cfg, out)
        else:
            ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=DEV)
            cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
            nsa.nsa_forward(d["q"], d["k"], d["v"], d["gates"], cfg, out)
        torch.cuda.synchronize()
        outs.append(out.float().cpu())
        idxs.append(idx.cpu())
    return outs, idxs


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    first = _problem(1, 1024, 4, 1, 64, 64, 4, 128, seed=0)           # the tiny workload
    second = _problem(1, 900, 64, 4, 192, 128, 16, 256, seed=3)      # a different layout in the same array
    for d, shape in (first, second):
        (ref, got), (ref_idx, got_idx) = _run_both(d, shape)
        assert torch.equal(ref_idx, got_idx)
        diff = (ref - got).abs()
        assert not torch.isnan(got).any()
        assert float(diff.max()) <= MAX_ABS and float(diff.mean()) <= MEAN_ABS


def test_noalloc_rejects_problems_beyond_its_scratch():
    d, shape = _problem(1, 256, 64, 4, 192, 128, 16, 256, seed=1)
    shape = dict(shape, seqlen=4096)          # needs about 134 MB of scratch, more than the 32 MiB built in
    cfg = nsa.make_config(w_cmp_k=d["w_k"], w_cmp_v=d["w_v"], **shape)
    assert nsa.nsa_workspace_size(cfg) > 32 << 20
    st = nsa.nsa_forward_noalloc(0x10000, 0x20000, 0x30000, 0x40000, cfg, 0x50000, check=False)
    assert st == nsa.NSA_ERR_WORKSPACE
    assert n_cmp(4096) == 255
