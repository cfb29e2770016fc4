"""nsa_forward_noalloc, the entry point for callers that cannot allocate device
memory (for instance a plugin whose host application owns every allocation):
through the C ABI its output and chosen blocks must equal, bit for bit, those of
nsa_forward (the entry point that takes a caller-allocated workspace; the two run
the same kernels on the same inputs, and the forward is deterministic), on calls
in a row with different problems sharing the same built-in scratch array.

The larger problem runs first, so the smaller one that follows finds the array
full of the previous call's values: nothing in it may need to start at zero.

This file is named so that pytest collects it last."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import synth
from block_sparse_attention_compress_b200 import build

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
            assert nsa.nsa_device_status_noalloc() == (nsa.NSA_OK, 0)
        else:
            ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=DEV)
            cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
            nsa.nsa_forward(d["q"], d["k"], d["v"], d["gates"], cfg, out)
            assert nsa.nsa_device_status(ws) == (nsa.NSA_OK, 0)
        torch.cuda.synchronize()
        outs.append(out.cpu())
        idxs.append(idx.cpu())
    return outs, idxs


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row():
    larger = _problem(1, 900, 64, 4, 192, 128, 16, 256, seed=3)      # fills most of the array
    tiny = _problem(1, 1024, 4, 1, 64, 64, 4, 128, seed=0)           # the tiny workload, a different layout
    for d, shape in (larger, tiny, larger):
        (ref, got), (ref_idx, got_idx) = _run_both(d, shape)
        assert not torch.isnan(got.float()).any()
        assert torch.equal(ref_idx, got_idx)
        assert torch.equal(ref, got)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """A problem that needs more scratch than the array holds is refused by status.  The
    tensors are real and of the problem's full size, so even a call that went ahead would
    touch only valid memory."""
    d, shape = _problem(1, 4096, 64, 4, 192, 128, 16, 256, seed=1)
    cfg = nsa.make_config(w_cmp_k=d["w_k"], w_cmp_v=d["w_v"], **shape)
    assert nsa.nsa_workspace_size(cfg) > 100 << 20      # about 134 MB of scratch
    out = torch.empty((1, 4096, 64, 128), dtype=torch.bfloat16, device=DEV)
    st = nsa.nsa_forward_noalloc(d["q"], d["k"], d["v"], d["gates"], cfg, out, check=False)
    torch.cuda.synchronize()
    assert st == nsa.NSA_ERR_WORKSPACE


def test_noalloc_rejects_dsa_mode():
    d, shape = _problem(1, 256, 16, 1, 192, 128, 16, 256, seed=2)
    cfg = nsa.make_config(mode=nsa.NSA_MODE_DSA, **shape)
    out = torch.empty((1, 256, 16, 128), dtype=torch.bfloat16, device=DEV)
    for call in (nsa.nsa_forward_noalloc, nsa.nsa_forward):
        assert call(d["q"], d["k"], d["v"], d["gates"], cfg, out, check=False) == nsa.NSA_ERR_INVALID_ARG
