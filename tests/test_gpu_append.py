"""nsa_compress_append: the compressed block each sequence's newest token completes, for a
growing decode cache.  It must equal bitwise the row the full compression computes (same
arithmetic, row by row) and the fp64 oracle's phi within bf16 rounding."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward
from tests.helpers import assert_close, assert_phi_close, idx_agreement

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def n_c(L):
    return 0 if L < 32 else (L - 32) // 16 + 1


@pytest.mark.parametrize("d", [192, 128, 64])
def test_append_rows_equal_full_compression(d):
    B, Lmax, H = 5, 1000, 4
    x = synth.decode_inputs(B, Lmax, 4 * H, H, d, d, seed=51)
    kx, w = x.k_cache.to(DEV), x.w_k.to(DEV)
    ncmax = n_c(Lmax)
    full = torch.empty((B, ncmax, H, d), dtype=torch.bfloat16, device=DEV)
    nsa.nsa_compress(kx, w, full)
    seqlens = torch.tensor([1000, 992, 32, 31, 48], dtype=torch.int32)
    app = torch.full((B, ncmax, H, d), -7.0, dtype=torch.bfloat16, device=DEV)
    nsa.nsa_compress_append(kx, w, seqlens.to(DEV), app)
    torch.cuda.synchronize()
    for b, L in enumerate(seqlens.tolist()):
        due = L >= 32 and (L - 32) % 16 == 0
        rows = torch.ones(ncmax, dtype=torch.bool)
        if due:
            i = (L - 32) // 16
            assert torch.equal(app[b, i], full[b, i]), (b, L)
            rows[i] = False
        assert torch.all(app[b][rows.to(DEV)] == -7.0), (b, L)   # nothing else written


def test_incremental_cache_equals_full_compression():
    """A decode loop that appends one token at a time and calls nsa_compress_append after
    each ends with the compressed cache of the full compression, bitwise, and within bf16
    rounding of the fp64 oracle."""
    B, L0, Lmax, H, d = 2, 100, 420, 2, 192
    x = synth.decode_inputs(B, Lmax, 8 * H, H, d, d, seed=52)
    kx, w = x.k_cache.to(DEV), x.w_k.to(DEV)
    ncmax = n_c(Lmax)
    kc = torch.zeros((B, ncmax, H, d), dtype=torch.bfloat16, device=DEV)
    prefix = torch.empty((B, n_c(L0), H, d), dtype=torch.bfloat16, device=DEV)
    nsa.nsa_compress(kx[:, :L0].contiguous(), w, prefix)     # the prefill's compressed cache
    kc[:, : n_c(L0)] = prefix
    for L in range(L0 + 1, Lmax + 1):   # token L-1 arrives
        nsa.nsa_compress_append(kx, w, torch.full((B,), L, dtype=torch.int32, device=DEV), kc)
    full = torch.empty_like(kc)
    nsa.nsa_compress(kx, w, full)
    torch.cuda.synchronize()
    assert torch.equal(kc, full)
    assert_phi_close(kc.cpu(), x.k_cache, x.w_k, "incremental kc")


# --------------------------------------------------------------------------
# phi as the two-layer MLP ([BLOG] "Deepseek 的论文核心点": an MLP compresses the blocks)
# --------------------------------------------------------------------------

def _mlp(d, seed):
    w1, b1, w2 = synth.phi_mlp_weights(32, d, seed=seed)
    return (w1, b1, w2), tuple(t.to(DEV) for t in (w1, b1, w2))


def _compress_mlp(x, wd):
    B, T, H, d = x.shape
    out = torch.empty((B, n_c(T), H, d), dtype=torch.bfloat16, device=DEV)
    hid = torch.empty_like(out)
    nsa.nsa_compress_mlp(x, *wd, hid, out)
    return out


@pytest.mark.parametrize("d", [192, 128, 64])
def test_compress_mlp_against_oracle(d):
    """nsa_compress_mlp against the oracle's MLP phi (hidden rounded to bf16 as stored):
    the same bounds as the forward's MLP caches."""
    B, T, H = 2, 700, 3
    x = synth.decode_inputs(B, T, 4 * H, H, d, d, seed=53)
    wc, wd = _mlp(d, seed=54)
    got = _compress_mlp(x.k_cache.to(DEV), wd)
    torch.cuda.synchronize()
    ref = oracle.compress_cache(x.k_cache, wc[0], 32, 16, True, (wc[1], wc[2]))
    assert_close(got.cpu(), ref, max_abs=3e-2, mean_abs=2e-3, what=f"mlp phi d={d}")


def test_compress_mlp_equals_forward_cache():
    """The compressed keys and values nsa_forward (phi_mlp = 1) writes to kc_out / vc_out are
    bitwise those nsa_compress_mlp computes: a decode cache built either way is the same."""
    B, T, hq, hkv, dk, dv = 1, 1001, 32, 2, 192, 128
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=55)
    (wk, bk, wk2), (wk_d, bk_d, wk2_d) = _mlp(dk, seed=56)
    (wv, bv, wv2), (wv_d, bv_d, wv2_d) = _mlp(dv, seed=57)
    f = NSAForward(B, T, hq, hkv, dk, dv, wk_d, wv_d, top_k=16, window=256,
                   mlp=dict(b_k=bk_d, w_k2=wk2_d, b_v=bv_d, w_v2=wv2_d))
    f(*[t.to(DEV) for t in (x.q, x.k, x.v, x.gates)])
    kc = _compress_mlp(x.k.to(DEV), (wk_d, bk_d, wk2_d))
    vc = _compress_mlp(x.v.to(DEV), (wv_d, bv_d, wv2_d))
    torch.cuda.synchronize()
    assert f.device_status() == 0
    assert torch.equal(kc, f.kc) and torch.equal(vc, f.vc)


@pytest.mark.parametrize("d", [192, 128, 64])
def test_append_mlp_rows_equal_full_compression(d):
    B, Lmax, H = 70, 400, 2     # more sequences than one 64-row tile
    x = synth.decode_inputs(B, Lmax, 4 * H, H, d, d, seed=58)
    kx = x.k_cache.to(DEV)
    _, wd = _mlp(d, seed=59)
    ncmax = n_c(Lmax)
    full = _compress_mlp(kx, wd)
    g = torch.Generator().manual_seed(60)
    seqlens = torch.randint(1, Lmax + 1, (B,), generator=g, dtype=torch.int32)
    seqlens[:6] = torch.tensor([400, 32, 31, 48, 1, 384], dtype=torch.int32)
    seqlens[6::3] = (32 + 16 * torch.randint(0, n_c(Lmax), (len(range(6, B, 3)),), generator=g)).to(torch.int32)
    app = torch.full((B, ncmax, H, d), -7.0, dtype=torch.bfloat16, device=DEV)
    hid = torch.empty((B, H, d), dtype=torch.bfloat16, device=DEV)
    nsa.nsa_compress_append_mlp(kx, *wd, seqlens.to(DEV), hid, app)
    torch.cuda.synchronize()
    n_due = 0
    for b, L in enumerate(seqlens.tolist()):
        rows = torch.ones(ncmax, dtype=torch.bool)
        if L >= 32 and (L - 32) % 16 == 0:
            i = (L - 32) // 16
            assert torch.equal(app[b, i], full[b, i]), (b, L)
            rows[i] = False
            n_due += 1
        assert torch.all(app[b][rows.to(DEV)] == -7.0), (b, L)   # nothing else written
    assert n_due >= B // 3


def test_mlp_cache_kept_by_append_then_decode():
    """A decode loop whose compressed caches use the MLP phi: prefill caches from
    nsa_compress_mlp, nsa_compress_append_mlp after every new token, then one nsa_decode step.
    The caches equal the full MLP compression bitwise, and the decode output matches the
    oracle's decode over the oracle's MLP caches."""
    B, L0, Lmax, hq, hkv, dk, dv = 2, 500, 700, 32, 2, 192, 128
    d = synth.decode_inputs(B, Lmax, hq, hkv, dk, dv, seed=61)
    (wk, bk, wk2), wkd = _mlp(dk, seed=62)
    (wv, bv, wv2), wvd = _mlp(dv, seed=63)
    k, v = d.k_cache.to(DEV), d.v_cache.to(DEV)
    ncmax = n_c(Lmax)
    kc = torch.zeros((B, ncmax, hkv, dk), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros((B, ncmax, hkv, dv), dtype=torch.bfloat16, device=DEV)
    kc[:, : n_c(L0)] = _compress_mlp(k[:, :L0].contiguous(), wkd)
    vc[:, : n_c(L0)] = _compress_mlp(v[:, :L0].contiguous(), wvd)
    hk = torch.empty((B, hkv, dk), dtype=torch.bfloat16, device=DEV)
    hv = torch.empty((B, hkv, dv), dtype=torch.bfloat16, device=DEV)
    lengths = torch.tensor([Lmax, Lmax - 37], dtype=torch.int32)
    for L in range(L0 + 1, Lmax + 1):   # token L-1 arrives; sequence 1 stops growing 37 tokens early
        sl = torch.minimum(lengths, torch.tensor(L, dtype=torch.int32)).to(DEV)
        nsa.nsa_compress_append_mlp(k, *wkd, sl, hk, kc)
        nsa.nsa_compress_append_mlp(v, *wvd, sl, hv, vc)
    torch.cuda.synchronize()
    for b, L in enumerate(lengths.tolist()):
        n = n_c(L)
        assert torch.equal(kc[b, :n], _compress_mlp(k[b:b + 1, :L].contiguous(), wkd)[0]), b
        assert torch.equal(vc[b, :n], _compress_mlp(v[b:b + 1, :L].contiguous(), wvd)[0]), b
    top_k, window = 16, 256
    idx = torch.full((B, hkv, top_k), -7, dtype=torch.int32, device=DEV)
    out = torch.empty((B, hq, dv), dtype=torch.bfloat16, device=DEV)
    cfg = nsa.make_config(batch=B, seqlen=Lmax, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=top_k, window=window,
                          w_cmp_k=wkd[0], w_cmp_v=wvd[0], sel_idx_out=idx)
    ws = torch.empty(max(nsa.nsa_workspace_size(cfg, B), 4), dtype=torch.uint8, device=DEV)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    nsa.nsa_decode(d.q.to(DEV), k, v, kc, vc, lengths.to(DEV), Lmax, d.gates.to(DEV), cfg, out)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a device-side wait timed out"
    kc_ref = oracle.compress_cache(d.k_cache, wk, 32, 16, True, (bk, wk2))
    vc_ref = oracle.compress_cache(d.v_cache, wv, 32, 16, True, (bv, wv2))
    ref = oracle.nsa_decode(d.q, d.k_cache, d.v_cache, kc_ref, vc_ref, lengths, d.gates, top_k=top_k, window=window)
    gi = idx.cpu()
    G = hq // hkv
    for b in range(B):
        for g in range(hkv):
            t = int(lengths[b]) - 1
            exact, swapped = idx_agreement(gi[b:b + 1, g:g + 1].unsqueeze(2), ref["idx"][b:b + 1, g:g + 1].unsqueeze(2),
                                           [[[ref["score"][b][g]]]], tokens=[t])
            if swapped:   # a legal near-tie swap: the oracle on the GPU's blocks for this group
                forced = oracle.nsa_decode(d.q, d.k_cache, d.v_cache, kc_ref, vc_ref, lengths, d.gates,
                                           top_k=top_k, window=window, batch=[b], forced_idx=gi[b:b + 1])
                ref["out"][b, g * G:(g + 1) * G] = forced["out"][0, g * G:(g + 1) * G]
    assert_close(out.cpu(), ref["out"], what="decode out over MLP caches")
