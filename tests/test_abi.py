"""The C-ABI library on the CPU: it loads, exports every entry point
include/nsa.h declares, its config struct matches the ctypes mirror, and
host-side validation answers without launching anything (no GPU needed)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import block_sparse_attention_compress_b200 as nsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nsa.h")


def _gpu_visible() -> bool:
    import torch
    return torch.cuda.is_available()


# The validation tests below hand the library made-up device addresses (or host memory) and
# expect a refusal before anything is launched.  They run only where no GPU can be reached, so
# that a future gap in the checks ends in a failed launch, never in a kernel on wild pointers.
made_up_pointers = pytest.mark.skipif(_gpu_visible(), reason="made-up device addresses: run where no GPU is visible")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_compress_b200 import build
    build.build()
    return nsa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(nsa.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", nsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(nsa_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


def test_config_layout_matches_header():
    src = r"""
    #include <stddef.h>
    #include <stdio.h>
    #include "nsa.h"
    int main(void) {
      printf("%zu", sizeof(nsa_config));
    #define F(x) printf(" %s=%zu", #x, offsetof(nsa_config, x));
      F(mode) F(batch) F(seqlen) F(h_q) F(h_kv) F(d_k) F(d_v) F(cmp_block) F(cmp_stride) F(sel_block)
      F(top_k) F(window) F(force_first) F(force_local) F(softmax_scale) F(w_cmp_k) F(w_cmp_v)
      F(sel_idx_out) F(kc_out) F(vc_out) F(workspace) F(workspace_bytes) F(stage_events) F(n_stage_events)
      F(score_map) F(phi_mlp) F(w_cmp_k2) F(w_cmp_v2) F(b_cmp_k) F(b_cmp_v)
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "l.c")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", os.path.join(d, "l")], check=True)
        got = subprocess.run([os.path.join(d, "l")], capture_output=True, text=True, check=True).stdout.split()
    assert int(got[0]) == ctypes.sizeof(nsa.NsaConfig)
    for item in got[1:]:
        name, off = item.split("=")
        assert getattr(nsa.NsaConfig, name).offset == int(off), name


def _cfg(**kw):
    base = dict(batch=1, seqlen=1024, h_q=4, h_kv=1, d_k=64, d_v=64, top_k=4, window=128,
                w_cmp_k=0x1000, w_cmp_v=0x2000)
    base.update(kw)
    return nsa.make_config(**base)


def test_status_strings(lib):
    for code, name in enumerate(["NSA_OK", "NSA_ERR_INVALID_ARG", "NSA_ERR_UNSUPPORTED", "NSA_ERR_WORKSPACE",
                                 "NSA_ERR_CUDA", "NSA_ERR_TIMEOUT"]):
        assert nsa.nsa_status_string(code) == name


def test_workspace_size_of_the_workloads(lib):
    c = _cfg()
    # status word and redo count, kc 63*64*2, vc same, idx 1*1024*4*4, acc 1024*4*64*4, the selected
    # branch's redo list 1*1*1024*4, a packed batch's checked cu_seqlens (B + 1)*4 (each rounded up
    # to 256 B)
    up = lambda x: (x + 255) // 256 * 256
    assert nsa.nsa_workspace_size(c) == (256 + 2 * up(63 * 64 * 2) + up(1024 * 4 * 4) + up(1024 * 4 * 64 * 4) +
                                         up(1024 * 4) + up(2 * 4))
    big = _cfg(seqlen=65536, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=16, window=512)
    assert nsa.nsa_workspace_size(big) > 65536 * 64 * 128 * 4
    assert nsa.nsa_workspace_size(_cfg(h_q=6, h_kv=4)) == 0
    # batch * seqlen * h_q rows up to 2^31 - 1 (32-bit row indices in the kernels), not beyond
    assert nsa.nsa_workspace_size(_cfg(batch=(1 << 31) // 4096 - 1)) > 0
    assert nsa.nsa_workspace_size(_cfg(batch=(1 << 31) // 4096)) == 0


@made_up_pointers
@pytest.mark.parametrize("kw,status", [
    (dict(h_q=6, h_kv=4), nsa.NSA_ERR_INVALID_ARG),
    (dict(batch=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(top_k=1), nsa.NSA_ERR_INVALID_ARG),            # fewer than the two forced blocks
    (dict(window=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(w_cmp_k=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(w_cmp_k=0x1004), nsa.NSA_ERR_INVALID_ARG),     # misaligned weights
    (dict(softmax_scale=-1.0), nsa.NSA_ERR_INVALID_ARG),
    (dict(mode=7), nsa.NSA_ERR_INVALID_ARG),
    (dict(sel_block=40), nsa.NSA_ERR_INVALID_ARG),       # not a multiple of the stride
    (dict(cmp_block=64, cmp_stride=32), nsa.NSA_ERR_UNSUPPORTED),
    (dict(h_q=32, h_kv=1), nsa.NSA_ERR_UNSUPPORTED),     # group of 32 heads
    (dict(d_k=96, d_v=96), nsa.NSA_ERR_UNSUPPORTED),
    (dict(seqlen=65537), nsa.NSA_ERR_UNSUPPORTED),
    (dict(top_k=33), nsa.NSA_ERR_UNSUPPORTED),
    (dict(batch=1 << 20, seqlen=1024, h_q=4), nsa.NSA_ERR_UNSUPPORTED),   # 2^32 (token, head) rows
])
def test_forward_rejects_bad_configs_without_launching(lib, kw, status):
    c = _cfg(**kw)
    st = nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0x40000, c, 0x50000, check=False)
    assert st == status


@made_up_pointers
def test_forward_rejects_null_and_misaligned_tensors(lib):
    c = _cfg(workspace=0x100000, workspace_bytes=1 << 30)
    assert nsa.nsa_forward(0, 0x20000, 0x30000, 0x40000, c, 0x50000, check=False) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_forward(0x10008, 0x20000, 0x30000, 0x40000, c, 0x50000, check=False) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0, c, 0x50000, check=False) == nsa.NSA_ERR_INVALID_ARG


@made_up_pointers
def test_forward_rejects_small_or_misaligned_workspace(lib):
    c = _cfg()
    need = nsa.nsa_workspace_size(c)
    for ws, nbytes in [(0, 0), (0x100000, need - 1), (0x100080, need)]:
        c.workspace, c.workspace_bytes = ws, nbytes
        st = nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0x40000, c, 0x50000, check=False)
        assert st == nsa.NSA_ERR_WORKSPACE


@made_up_pointers
def test_compress_rejects_bad_arguments(lib):
    L = lib
    assert L.nsa_compress(0, 0x1000, 1, 64, 1, 64, 64, 32, 16, 0x2000, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress(0x1000, 0x2000, 1, 64, 1, 64, 64, 16, 8, 0x3000, None) == nsa.NSA_ERR_UNSUPPORTED
    assert L.nsa_compress(0x1000, 0x2000, 1, 64, 1, 96, 96, 32, 16, 0x3000, None) == nsa.NSA_ERR_UNSUPPORTED
    assert L.nsa_compress(0x1000, 0x2000, 0, 64, 1, 64, 64, 32, 16, 0x3000, None) == nsa.NSA_ERR_INVALID_ARG


@made_up_pointers
def test_compress_mlp_rejects_bad_arguments(lib):
    """Argument checks of the MLP phi entry points, all before any CUDA call."""
    L = lib
    a, b, c, d, h, o = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000
    assert L.nsa_compress_mlp(a, b, 0, d, 1, 64, 1, 64, 32, 16, h, o, None) == nsa.NSA_ERR_INVALID_ARG  # no bias
    assert L.nsa_compress_mlp(a, b, c, d, 1, 64, 1, 64, 32, 16, 0, o, None) == nsa.NSA_ERR_INVALID_ARG  # no hidden
    assert L.nsa_compress_mlp(a, b, c + 8, d, 1, 64, 1, 64, 32, 16, h, o, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_mlp(a, b, c, d, 1, 64, 1, 96, 32, 16, h, o, None) == nsa.NSA_ERR_UNSUPPORTED
    assert L.nsa_compress_mlp(a, b, c, d, 1, 64, 1, 64, 16, 8, h, o, None) == nsa.NSA_ERR_UNSUPPORTED
    sl = 0x7000
    assert L.nsa_compress_append_mlp(a, b, c, d, sl, 2, 64, 1, 64, 32, 16, 0, o, 3, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_append_mlp(a, b, c, d, sl + 2, 2, 64, 1, 64, 32, 16, h, o, 3, None) == \
        nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_append_mlp(a, b, c, d, sl, 2, 64, 1, 64, 32, 16, h, o, 0, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_append_mlp(a, b, c, d, sl, 2, 64, 1, 192, 16, 16, h, o, 3, None) == \
        nsa.NSA_ERR_UNSUPPORTED


@made_up_pointers
def test_backward_entry_points_check_their_arguments(lib):
    """nsa_backward takes the linear phi only; nsa_backward_ex needs the MLP's gradient buffers
    when phi is the MLP.  All checked before any CUDA call."""
    c = _cfg(h_q=16, h_kv=1, d_k=192, d_v=128)
    c.phi_mlp, c.w_cmp_k2, c.w_cmp_v2, c.b_cmp_k, c.b_cmp_v = 1, 0x7000, 0x8000, 0x9000, 0xa000
    p = [0x10000 * (i + 1) for i in range(12)]
    st = lib.nsa_backward(p[0], p[1], p[2], p[3], p[4], p[5], ctypes.byref(c), p[6], p[7], p[8], p[9], p[10], p[11],
                          None)
    assert st == nsa.NSA_ERR_UNSUPPORTED
    g = nsa.NsaGrads(dq=p[6], dk=p[7], dv=p[8], dgates=p[9], dw_k=p[10], dw_v=p[11])   # no MLP gradients
    st = lib.nsa_backward_ex(p[0], p[1], p[2], p[3], p[4], p[5], None, 0, ctypes.byref(c), ctypes.byref(g), None)
    assert st == nsa.NSA_ERR_INVALID_ARG
    assert lib.nsa_backward_ex(p[0], p[1], p[2], p[3], p[4], p[5], None, 0, ctypes.byref(c), None, None) == \
        nsa.NSA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(nsa, "_lib", None)
    monkeypatch.setattr(nsa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        nsa.load_library()


@made_up_pointers
def test_status_and_selftest_reject_bad_arguments(lib):
    """Argument checks that return before any CUDA call (safe without a GPU)."""
    word = ctypes.c_int32(7)
    assert lib.nsa_device_status(None, ctypes.byref(word), None) == nsa.NSA_ERR_INVALID_ARG
    assert lib.nsa_selftest_wait_timeout(None, 256, 1000, None) == nsa.NSA_ERR_INVALID_ARG
    fake = 0x10000   # never dereferenced: every call below fails its checks first
    assert lib.nsa_selftest_wait_timeout(fake, 2, 1000, None) == nsa.NSA_ERR_INVALID_ARG          # too small
    assert lib.nsa_selftest_wait_timeout(fake + 2, 256, 1000, None) == nsa.NSA_ERR_INVALID_ARG    # misaligned
    assert lib.nsa_selftest_wait_timeout(fake, 256, 0, None) == nsa.NSA_ERR_INVALID_ARG           # no limit
    assert lib.nsa_selftest_wait_timeout(fake, 256, 1000001, None) == nsa.NSA_ERR_INVALID_ARG     # above 1 s


@made_up_pointers
def test_compress_append_rejects_bad_arguments(lib):
    f = 0x10000   # never dereferenced: every call below fails its checks first
    ok_args = dict(x=f, w=f, sl=f, B=2, L=64, H=1, d=64, dout=64, l=32, s=16, out=f, nc=3)

    def call(**kw):
        a = dict(ok_args, **kw)
        return lib.nsa_compress_append(a["x"], a["w"], a["sl"], a["B"], a["L"], a["H"], a["d"], a["dout"], a["l"],
                                       a["s"], a["out"], a["nc"], None)
    assert call(x=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(sl=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(sl=f + 2) == nsa.NSA_ERR_INVALID_ARG      # seqlens misaligned
    assert call(out=f + 8) == nsa.NSA_ERR_INVALID_ARG     # cache misaligned
    assert call(nc=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(l=64) == nsa.NSA_ERR_UNSUPPORTED
    assert call(d=96, dout=96) == nsa.NSA_ERR_UNSUPPORTED


@made_up_pointers
def test_forward_varlen_rejects_bad_arguments(lib):
    """Checks that return before any CUDA call (safe without a GPU): pointers, the packed row
    count, the mode, and the shapes the tensor-core kernels do not take."""
    f = 0x10000   # never dereferenced: every call below fails its checks first

    def call(c, cu=f, total=100, q=f, gates=f):
        return lib.nsa_forward_varlen(q, f, f, gates, cu, total, ctypes.byref(c), f, None)

    c = _cfg(h_q=16, h_kv=1, d_k=192, d_v=128, batch=2, seqlen=64, workspace=0x100000, workspace_bytes=1 << 30)
    assert call(c, cu=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(c, cu=f + 2) == nsa.NSA_ERR_INVALID_ARG            # misaligned offsets
    assert call(c, gates=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(c, q=f + 8) == nsa.NSA_ERR_INVALID_ARG             # misaligned q
    assert call(c, total=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(c, total=129) == nsa.NSA_ERR_INVALID_ARG           # more rows than batch x seqlen
    small = _cfg(h_q=4, h_kv=1, d_k=64, d_v=64, batch=2, seqlen=64, workspace=0x100000, workspace_bytes=1 << 30)
    assert call(small, total=64) == nsa.NSA_ERR_UNSUPPORTED        # the warp-MMA shapes
    moba = _cfg(mode=nsa.NSA_MODE_MOBA, h_q=2, h_kv=2, d_k=128, d_v=128, sel_block=64, top_k=3, w_cmp_k=0,
                w_cmp_v=0, batch=1, seqlen=128)
    assert call(moba, total=64) == nsa.NSA_ERR_UNSUPPORTED
    c.workspace_bytes = 16
    assert call(c, total=64) == nsa.NSA_ERR_WORKSPACE


@made_up_pointers
def test_unknown_score_map_is_rejected(lib):
    c = _cfg(score_map=3)
    assert nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0x40000, c, 0x50000, check=False) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_workspace_size(_cfg(score_map=-1)) == 0


@made_up_pointers
def test_phi_mlp_needs_its_weights(lib):
    base = dict(workspace=0x100000, workspace_bytes=1 << 30)
    assert nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0x40000, _cfg(phi_mlp=1, **base), 0x50000,
                           check=False) == nsa.NSA_ERR_INVALID_ARG
    misaligned = _cfg(phi_mlp=1, w_cmp_k2=0x3000, w_cmp_v2=0x4000, b_cmp_k=0x5008, b_cmp_v=0x6000, **base)
    assert nsa.nsa_forward(0x10000, 0x20000, 0x30000, 0x40000, misaligned, 0x50000,
                           check=False) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_workspace_size(_cfg(phi_mlp=2)) == 0
    lin = nsa.nsa_workspace_size(_cfg())
    mlp = nsa.nsa_workspace_size(_cfg(phi_mlp=1, w_cmp_k2=0x3000, w_cmp_v2=0x4000, b_cmp_k=0x5000, b_cmp_v=0x6000))
    assert mlp > lin   # the hidden rows


@made_up_pointers
def test_backward_rejects_bad_arguments(lib):
    f = 0x10000   # never dereferenced: every call below fails its checks first
    base = dict(workspace=0x100000, workspace_bytes=1 << 30)

    def call(c, **kw):
        a = dict(q=f, k=f, v=f, gates=f, sel=f, dout=f, dq=f, dk=f, dv=f, dg=f, dwk=f, dwv=f)
        a.update(kw)
        return lib.nsa_backward(a["q"], a["k"], a["v"], a["gates"], a["sel"], a["dout"], ctypes.byref(c), a["dq"],
                                a["dk"], a["dv"], a["dg"], a["dwk"], a["dwv"], None)

    c = _cfg(**base)
    assert call(c, sel=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(c, dout=f + 8) == nsa.NSA_ERR_INVALID_ARG
    assert call(c, dg=f + 2) == nsa.NSA_ERR_INVALID_ARG
    mlp = _cfg(phi_mlp=1, w_cmp_k2=0x3000, w_cmp_v2=0x4000, b_cmp_k=0x5000, b_cmp_v=0x6000, **base)
    assert call(mlp) == nsa.NSA_ERR_UNSUPPORTED
    moba = _cfg(mode=nsa.NSA_MODE_MOBA, h_q=2, h_kv=2, d_k=128, d_v=128, sel_block=64, top_k=3, w_cmp_k=0,
                w_cmp_v=0, **base)
    assert call(moba) == nsa.NSA_ERR_UNSUPPORTED
    c.workspace_bytes = 16
    assert call(c) == nsa.NSA_ERR_WORKSPACE


def test_dsa_workspace_holds_only_the_chosen_tokens(lib):
    """DSA keeps no score matrix: the status word and the [B, T, top_k] chosen tokens."""
    up = lambda n: (n + 255) // 256 * 256
    for B, T, K in [(1, 8192, 2048), (2, 32768, 2048), (1, 131072, 512)]:
        c = nsa.make_config(mode=nsa.NSA_MODE_DSA, batch=B, seqlen=T, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=K)
        assert nsa.nsa_workspace_size(c) == 256 + up(B * T * K * 4), (B, T, K)
    c = nsa.make_config(mode=nsa.NSA_MODE_DSA, batch=1, seqlen=131073, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=64)
    assert nsa.nsa_workspace_size(c) == 0   # past the supported length


@made_up_pointers
def test_forward_rejects_dsa_mode(lib):
    """DSA has its own entry point; nsa_forward and nsa_forward_noalloc refuse its mode
    before anything runs (real host tensors, never dereferenced)."""
    import torch
    t = [torch.zeros(4096, dtype=torch.uint8) for _ in range(6)]
    c = _cfg(mode=nsa.NSA_MODE_DSA, h_q=16, h_kv=1, d_k=192, d_v=128, top_k=16, cmp_stride=0,
             workspace=t[5].data_ptr(), workspace_bytes=1 << 30)
    assert nsa.nsa_forward(t[0], t[1], t[2], t[3], c, t[4], check=False) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_forward_noalloc(t[0], t[1], t[2], t[3], c, t[4], check=False) == nsa.NSA_ERR_INVALID_ARG
