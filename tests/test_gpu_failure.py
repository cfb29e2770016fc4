"""The failure path of the bounded device-side waits, on the GPU without a fault: a wait
that nothing releases gives up after its limit, the status word reports it through
nsa_device_status, and the context stays usable for the next forward."""
import pytest
import torch

import block_sparse_attention_compress_b200 as nsa
import synth
from block_sparse_attention_compress_b200 import build
from block_sparse_attention_compress_b200.torch_ops import NSAForward

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def test_wait_that_nothing_releases_reports_timeout():
    ws = torch.full((256,), 0x55, dtype=torch.uint8, device=DEV)
    nsa.nsa_selftest_wait_timeout(ws, 20000)          # 20 ms limit
    st, word = nsa.nsa_device_status(ws)
    assert st == nsa.NSA_ERR_TIMEOUT and word == 99
    assert torch.all(ws[4:] == 0x55)                  # nothing but the status word is written


def test_context_usable_after_timeout_and_status_clean():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    nsa.nsa_selftest_wait_timeout(ws, 5000)
    assert nsa.nsa_device_status(ws) == (nsa.NSA_ERR_TIMEOUT, 99)
    x = synth.nsa_inputs(1, 300, 16, 1, 192, 128, seed=41)
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.gates, x.w_k, x.w_v)]
    f = NSAForward(1, 300, 16, 1, 192, 128, dev[4], dev[5], top_k=8, window=64)
    out = f(*dev[:4])
    assert nsa.nsa_device_status(f.workspace) == (nsa.NSA_OK, 0)
    assert torch.isfinite(out.float()).all()
