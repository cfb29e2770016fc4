"""nsa_compress_append: the compressed block each sequence's newest token completes, for a
growing decode cache.  It must equal bitwise the row the full compression computes (same
arithmetic, row by row) and the fp64 oracle's phi within bf16 rounding."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import oracle
import synth
from block_sparse_attention_compress_b200 import build
from tests.helpers import assert_phi_close

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
