"""GPU parity of the NSA backward (nsa_backward) against torch autograd through the fp64
oracle forward, run with the blocks the GPU forward chose (forced-index mode: the choice is
discrete and carries no gradient)."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL = 2e-2   # relative L2 error per gradient (bf16 operands, fp32 accumulation)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def rel_err(got, ref):
    return float((got.double() - ref).norm() / ref.norm().clamp_min(1e-30))


@pytest.mark.parametrize("shape,top_k,window", [
    ((1, 200, 16, 1, 192, 128), 4, 96),     # one group of 16 heads, ragged blocks
    ((2, 150, 8, 2, 64, 64), 3, 40),        # two groups of 4 heads, batch 2
    ((1, 520, 16, 1, 192, 128), 8, 300),    # several 16-row tiles per warp in the selected and window branches
])
def test_backward_matches_autograd(shape, top_k, window):
    B, T, hq, hkv, dk, dv = shape
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=81)
    g = torch.Generator().manual_seed(82)
    dout = torch.randn(B, T, hq, dv, generator=g).to(torch.bfloat16)
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.gates, x.w_k, x.w_v, dout)]
    f = NSAForward(B, T, hq, hkv, dk, dv, dev[4], dev[5], top_k=top_k, window=window)
    f(*dev[:4])
    grads = dict(dq=torch.empty(B, T, hq, dk), dk=torch.empty(B, T, hkv, dk), dv=torch.empty(B, T, hkv, dv),
                 dgates=torch.empty(B, T, hq, 3), dw_k=torch.empty(32 * dk, dk), dw_v=torch.empty(32 * dv, dv))
    gd = {n: t.to(DEV) for n, t in grads.items()}
    nsa.nsa_backward(dev[0], dev[1], dev[2], dev[3], f.idx, dev[6], f.cfg, gd["dq"], gd["dk"], gd["dv"], gd["dgates"],
                     gd["dw_k"], gd["dw_v"])
    torch.cuda.synchronize()
    idx = f.idx.cpu()
    leaves = {n: t.double().requires_grad_() for n, t in
              (("q", x.q), ("k", x.k), ("v", x.v), ("gates", x.gates), ("w_k", x.w_k), ("w_v", x.w_v))}
    ref = oracle.nsa_forward(leaves["q"], leaves["k"], leaves["v"], leaves["gates"], leaves["w_k"], leaves["w_v"],
                             top_k=top_k, window=window, forced_idx=idx)
    (ref["out"] * dout.double()).sum().backward()
    pairs = dict(dq="q", dk="k", dv="v", dgates="gates", dw_k="w_k", dw_v="w_v")
    for name, leaf in pairs.items():
        err = rel_err(gd[name].cpu(), leaves[leaf].grad)
        assert err <= REL, f"{name}: relative error {err:.2e}"
