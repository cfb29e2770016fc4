"""GPU parity of the NSA backward (nsa_backward) against torch autograd through the fp64
oracle forward, run with the blocks the GPU forward chose (forced-index mode: the choice is
discrete and carries no gradient)."""
import dataclasses

import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward, NSAForwardVarlen

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_REL = 2e-2    # per gradient tensor: max |err| <= MAX_REL * max |ref|  (bf16 operands, fp32 accumulation)
MEAN_REL = 2e-3   #                      mean |err| <= MEAN_REL * max |ref|


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def assert_grad_close(name, got, ref):
    """Element by element: every entry within MAX_REL of the tensor's largest reference entry,
    and the mean error within MEAN_REL of it."""
    ref = ref.detach().double()
    err = (got.detach().cpu().double() - ref).abs()
    scale = float(ref.abs().max())
    assert scale > 0, name
    mx, mn = float(err.max()), float(err.mean())
    print(f"{name}: max {mx / scale:.2e} mean {mn / scale:.2e} of max|ref| {scale:.3e}")
    assert mx <= MAX_REL * scale and mn <= MEAN_REL * scale, \
        f"{name}: max {mx:.3e} mean {mn:.3e} against max|ref| {scale:.3e}"


def run_and_compare(x, dout, top_k, window, tokens=None, mlp=None):
    """GPU forward (for the chosen blocks) and backward through the C ABI; the oracle's fp64
    autograd through its forward at ``tokens`` (all if None; dout must be zero elsewhere) in
    forced-index mode on the GPU's choice; every gradient compared element by element.
    ``mlp`` = dict(b_k, w_k2, b_v, w_v2) (host tensors) makes phi the two-layer MLP, with
    x.w_k / x.w_v as its first layers; the backward then runs through nsa_backward_ex."""
    B, T, hq, dk = x.q.shape
    hkv, dv = x.k.shape[2], x.v.shape[3]
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.gates, x.w_k, x.w_v, dout)]
    mlp_dev = None if mlp is None else {n: t.to(DEV) for n, t in mlp.items()}
    f = NSAForward(B, T, hq, hkv, dk, dv, dev[4], dev[5], top_k=top_k, window=window, mlp=mlp_dev)
    f(*dev[:4])
    grads = dict(dq=torch.empty(B, T, hq, dk), dk=torch.empty(B, T, hkv, dk), dv=torch.empty(B, T, hkv, dv),
                 dgates=torch.empty(B, T, hq, 3), dw_k=torch.empty(32 * dk, dk), dw_v=torch.empty(32 * dv, dv))
    if mlp is not None:
        grads.update(db_k=torch.empty(dk), db_v=torch.empty(dv), dw_k2=torch.empty(dk, dk), dw_v2=torch.empty(dv, dv))
    gd = {n: t.to(DEV) for n, t in grads.items()}
    if mlp is None:
        nsa.nsa_backward(dev[0], dev[1], dev[2], dev[3], f.idx, dev[6], f.cfg, gd["dq"], gd["dk"], gd["dv"],
                         gd["dgates"], gd["dw_k"], gd["dw_v"])
    else:
        nsa.nsa_backward_ex(dev[0], dev[1], dev[2], dev[3], f.idx, dev[6], f.cfg, gd)
    torch.cuda.synchronize()
    assert f.device_status() == 0
    idx = f.idx.cpu()
    toks = list(range(T)) if tokens is None else list(tokens)
    named = [("q", x.q), ("k", x.k), ("v", x.v), ("gates", x.gates), ("w_k", x.w_k), ("w_v", x.w_v)]
    if mlp is not None:
        named += list(mlp.items())
    leaves = {n: t.double().requires_grad_() for n, t in named}
    ref = oracle.nsa_forward(leaves["q"], leaves["k"], leaves["v"], leaves["gates"], leaves["w_k"], leaves["w_v"],
                             top_k=top_k, window=window, tokens=toks, forced_idx=idx[:, :, toks],
                             mlp=None if mlp is None else {n: leaves[n] for n in mlp})
    (ref["out"] * dout[:, toks].double()).sum().backward()
    pairs = dict(dq="q", dk="k", dv="v", dgates="gates", dw_k="w_k", dw_v="w_v")
    if mlp is not None:
        pairs.update(db_k="b_k", db_v="b_v", dw_k2="w_k2", dw_v2="w_v2")
    for name, leaf in pairs.items():
        assert_grad_close(name, gd[name], leaves[leaf].grad)


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
    run_and_compare(x, dout, top_k, window)


def test_backward_8k_workload_sampled_rows():
    """The 8K workload the benchmark times (64 query heads in 4 groups, d_k 192, d_v 128,
    top-16, window 512) with dout nonzero on sampled rows only: every gradient then depends on
    those rows alone, so the oracle's autograd over the sampled tokens gives all of dq, dk, dv,
    dgates, dW_k and dW_v, each compared element by element."""
    c = synth.WORKLOADS["nsa_8k"]
    B, T, hq, hkv, dk, dv = c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=0)
    g = torch.Generator().manual_seed(83)
    toks = sorted(set([0, 31, 64, 511, 512, 4096, T - 1] + torch.randint(0, T, (17,), generator=g).tolist()))
    dout = torch.zeros(B, T, hq, dv)
    dout[:, toks] = torch.randn(B, len(toks), hq, dv, generator=g)
    run_and_compare(x, dout.to(torch.bfloat16), c["top_k"], c["window"], tokens=toks)


@pytest.mark.parametrize("shape,top_k,window", [
    ((1, 300, 16, 1, 192, 128), 4, 96),     # the tensor-core forward shapes
    ((2, 150, 8, 2, 64, 64), 3, 40),        # two groups of 4 heads, batch 2
])
def test_backward_mlp_phi_matches_autograd(shape, top_k, window):
    """phi as the two-layer MLP ([BLOG] "Deepseek 的论文核心点"): the gradients of q, k, v, the
    gates and both layers' weights and first-layer bias, through nsa_backward_ex."""
    B, T, hq, hkv, dk, dv = shape
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=84)
    w_k, b_k, w_k2 = synth.phi_mlp_weights(32, dk, seed=85)
    w_v, b_v, w_v2 = synth.phi_mlp_weights(32, dv, seed=86)
    x = dataclasses.replace(x, w_k=w_k, w_v=w_v)
    g = torch.Generator().manual_seed(87)
    dout = torch.randn(B, T, hq, dv, generator=g).to(torch.bfloat16)
    run_and_compare(x, dout, top_k, window, mlp=dict(b_k=b_k, w_k2=w_k2, b_v=b_v, w_v2=w_v2))



@pytest.mark.parametrize("lengths,mlp", [
    ([200, 1, 33, 0, 150], False),   # ragged, a single token, shorter than a compression block, empty
    ([130, 77], True),               # with the MLP phi
])
def test_backward_varlen_matches_autograd(lengths, mlp):
    """A packed variable-length batch through nsa_backward_ex: the oracle runs each sequence
    alone (forced to the GPU forward's blocks) on slices of the packed leaves, so its autograd
    gives the packed dq, dk, dv and dgates and the weight gradients summed over the sequences."""
    hq, hkv, dk, dv, top_k, window = 16, 1, 192, 128, 4, 96
    x, cu = synth.nsa_varlen_inputs(lengths, hq, hkv, dk, dv, seed=91)
    mw = None
    if mlp:
        w_k, b_k, w_k2 = synth.phi_mlp_weights(32, dk, seed=92)
        w_v, b_v, w_v2 = synth.phi_mlp_weights(32, dv, seed=93)
        x = dataclasses.replace(x, w_k=w_k, w_v=w_v)
        mw = dict(b_k=b_k, w_k2=w_k2, b_v=b_v, w_v2=w_v2)
    B, T, total = len(lengths), max(lengths), int(cu[-1])
    g = torch.Generator().manual_seed(94)
    dout = torch.randn(total, hq, dv, generator=g).to(torch.bfloat16)
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.gates, x.w_k, x.w_v, dout, cu)]
    f = NSAForwardVarlen(B, T, hq, hkv, dk, dv, dev[4], dev[5], top_k=top_k, window=window,
                         mlp=None if mw is None else {n: t.to(DEV) for n, t in mw.items()})
    f(*dev[:4], dev[7])
    grads = dict(dq=torch.empty(total, hq, dk), dk=torch.empty(total, hkv, dk), dv=torch.empty(total, hkv, dv),
                 dgates=torch.empty(total, hq, 3), dw_k=torch.empty(32 * dk, dk), dw_v=torch.empty(32 * dv, dv))
    if mlp:
        grads.update(db_k=torch.empty(dk), db_v=torch.empty(dv), dw_k2=torch.empty(dk, dk), dw_v2=torch.empty(dv, dv))
    gd = {n: t.to(DEV) for n, t in grads.items()}
    nsa.nsa_backward_ex(dev[0], dev[1], dev[2], dev[3], f.idx, dev[6], f.cfg, gd, cu_seqlens=dev[7])
    torch.cuda.synchronize()
    assert f.device_status() == 0
    idx = f.idx.cpu()
    named = [("q", x.q), ("k", x.k), ("v", x.v), ("gates", x.gates), ("w_k", x.w_k), ("w_v", x.w_v)]
    if mlp:
        named += list(mw.items())
    leaves = {n: t.double().requires_grad_() for n, t in named}
    loss = 0.0
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        lo = int(cu[b])
        sl = lambda n: leaves[n][lo:lo + L].unsqueeze(0)
        ref = oracle.nsa_forward(sl("q"), sl("k"), sl("v"), sl("gates"), leaves["w_k"], leaves["w_v"],
                                 top_k=top_k, window=window, forced_idx=idx[b:b + 1, :, :L],
                                 mlp=None if mw is None else {n: leaves[n] for n in mw})
        loss = loss + (ref["out"][0] * dout[lo:lo + L].double()).sum()
    loss.backward()
    pairs = dict(dq="q", dk="k", dv="v", dgates="gates", dw_k="w_k", dw_v="w_v")
    if mlp:
        pairs.update(db_k="b_k", db_v="b_v", dw_k2="w_k2", dw_v2="w_v2")
    for name, leaf in pairs.items():
        assert_grad_close(name, gd[name], leaves[leaf].grad)
