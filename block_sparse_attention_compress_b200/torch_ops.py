"""Torch-facing convenience calls over the C ABI: they allocate the outputs
and the workspace with torch (device memory is all torch provides) and call
the library's entry points on the current stream."""
from __future__ import annotations

import torch

from . import (NSA_MODE_MOBA, NSA_MODE_NSA, make_config, nsa_compress, nsa_decode, nsa_forward,
               nsa_forward_varlen, nsa_workspace_size)


def n_cmp(T: int, l: int = 32, s: int = 16) -> int:
    return 0 if T < l else (T - l) // s + 1


class NSAForward:
    """Prefill forward with a reusable workspace (one allocation per shape)."""

    def __init__(self, B, T, h_q, h_kv, d_k, d_v, w_k, w_v, *, top_k=16, window=512, sel_block=64,
                 force_first=1, force_local=1, softmax_scale=0.0, keep_idx=True, keep_kc=True, device="cuda",
                 score_map=0, mlp=None):
        """mlp: dict(b_k, w_k2, b_v, w_v2) of device tensors makes phi the two-layer MLP (w_k and
        w_v are then its first layers); None keeps the linear phi."""
        self.shape = (B, T, h_q, h_kv, d_k, d_v)
        nc = n_cmp(T)
        self.idx = torch.empty((B, h_kv, T, top_k), dtype=torch.int32, device=device) if keep_idx else None
        self.kc = torch.empty((B, nc, h_kv, d_k), dtype=torch.bfloat16, device=device) if keep_kc else None
        self.vc = torch.empty((B, nc, h_kv, d_v), dtype=torch.bfloat16, device=device) if keep_kc else None
        self.w_k, self.w_v = w_k, w_v
        self.cfg = make_config(mode=NSA_MODE_NSA, batch=B, seqlen=T, h_q=h_q, h_kv=h_kv, d_k=d_k, d_v=d_v,
                               top_k=top_k, window=window, sel_block=sel_block, force_first=force_first,
                               force_local=force_local, softmax_scale=softmax_scale, w_cmp_k=w_k, w_cmp_v=w_v,
                               sel_idx_out=self.idx, kc_out=self.kc, vc_out=self.vc, score_map=score_map)
        if mlp is not None:
            self.mlp = mlp   # keep the weights alive as long as the config points at them
            for name, val in (("phi_mlp", 1), ("w_cmp_k2", mlp["w_k2"].data_ptr()), ("w_cmp_v2", mlp["w_v2"].data_ptr()),
                              ("b_cmp_k", mlp["b_k"].data_ptr()), ("b_cmp_v", mlp["b_v"].data_ptr())):
                setattr(self.cfg, name, val)
        nbytes = nsa_workspace_size(self.cfg)
        if nbytes == 0:
            raise ValueError("nsa_workspace_size rejected the configuration")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.cfg.workspace = self.workspace.data_ptr()
        self.cfg.workspace_bytes = nbytes

    def device_status(self) -> int:
        """The workspace's status word after a synchronised call: 0, or the code of a
        device-side wait that timed out."""
        return int(self.workspace[:4].view(torch.int32).item())

    def __call__(self, q, k, v, gates, out=None):
        B, T, h_q, h_kv, d_k, d_v = self.shape
        if out is None:
            out = torch.empty((B, T, h_q, d_v), dtype=torch.bfloat16, device=q.device)
        nsa_forward(q, k, v, gates, self.cfg, out)
        return out


class NSAForwardVarlen(NSAForward):
    """Prefill forward of a packed batch of sequences of different lengths (at most T
    tokens each): q [total, h_q, d_k], k/v [total, h_kv, d], gates [total, h_q, 3], and
    cu_seqlens int32 [B + 1] on the device.  idx, kc and vc keep the per-sequence layouts of
    NSAForward (B sequences of up to T tokens)."""

    def __call__(self, q, k, v, gates, cu_seqlens, out=None):
        B, T, h_q, h_kv, d_k, d_v = self.shape
        if out is None:
            out = torch.empty((q.shape[0], h_q, d_v), dtype=torch.bfloat16, device=q.device)
        nsa_forward_varlen(q, k, v, gates, cu_seqlens, self.cfg, out)
        return out


def nsa_forward_torch(q, k, v, gates, w_k, w_v, **kw):
    """One-shot forward: returns (out, idx, kc, vc)."""
    B, T, h_q, d_k = q.shape
    h_kv, d_v = k.shape[2], v.shape[3]
    f = NSAForward(B, T, h_q, h_kv, d_k, d_v, w_k, w_v, device=q.device, **kw)
    out = f(q, k, v, gates)
    return out, f.idx, f.kc, f.vc


def compress_torch(x, w, l=32, s=16):
    B, T, H, d = x.shape
    out = torch.empty((B, n_cmp(T, l, s), H, w.shape[1]), dtype=torch.bfloat16, device=x.device)
    if out.shape[1]:
        nsa_compress(x, w, out, l, s)
    return out
