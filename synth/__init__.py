"""Seeded synthetic inputs for the NSA and MoBA workloads.

This module only draws random tensors; it holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can consume its output
without sharing any of the method's code.

Recipe (one ``torch.Generator`` per call, seeded, draws in this fixed order):

  q       ~ N(0, 1)                         [B, T, H_q, d_k]
  k       ~ N(0, 1) + offset[t // 64]       [B, T, H_kv, d_k]
  offset  ~ N(0, 0.5^2)                     [B, ceil(T/64), H_kv, d_k]
  v       ~ N(0, 1)                         [B, T, H_kv, d_v]
  W_k     ~ N(0, 1/(l*d_k))                 [l*d_k, d_k]   (NSA only)
  W_v     ~ N(0, 1/(l*d_v))                 [l*d_v, d_v]   (NSA only)
  gates   = sigmoid(N(0, 1))                [B, T, H_q, 3] (NSA only; order cmp, slc, win)

Every tensor is drawn in fp32 and rounded once to bf16 (round to nearest
even); the key offsets are added before that rounding.  The draw order is
q, k-noise, offsets, v, W_k, W_v, gate logits, whatever the device.  The
same seed on a different device gives different (but equally distributed)
numbers: the CPU generator is the canonical one for anything the oracle
checks element by element; the CUDA generator only serves large timing
runs and sampled parity checks (whose oracle inputs are copied back from
those very tensors).
"""
from __future__ import annotations

import dataclasses
import math

import torch

OFFSET_BLOCK = 64      # tokens that share one key offset vector
OFFSET_STD = 0.5


@dataclasses.dataclass
class NSAInputs:
    q: torch.Tensor          # [B, T, H_q, d_k] bf16
    k: torch.Tensor          # [B, T, H_kv, d_k] bf16
    v: torch.Tensor          # [B, T, H_kv, d_v] bf16
    w_k: torch.Tensor        # [l*d_k, d_k] bf16
    w_v: torch.Tensor        # [l*d_v, d_v] bf16
    gates: torch.Tensor      # [B, T, H_q, 3] bf16


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor          # [B, H_q, d_k] bf16 (the query at position L-1)
    k_cache: torch.Tensor    # [B, L, H_kv, d_k] bf16 (includes the new token)
    v_cache: torch.Tensor    # [B, L, H_kv, d_v] bf16
    w_k: torch.Tensor
    w_v: torch.Tensor
    gates: torch.Tensor      # [B, H_q, 3] bf16
    seqlens: torch.Tensor    # [B] int32


@dataclasses.dataclass
class MobaInputs:
    q: torch.Tensor          # [B, T, H, d] bf16
    k: torch.Tensor          # [B, T, H, d] bf16
    v: torch.Tensor          # [B, T, H, d] bf16


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, device, std=1.0):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def _keys(g, B, T, H, d, device):
    """Key noise plus one offset vector per 64-token block (same draw order everywhere)."""
    noise = _randn(g, (B, T, H, d), device)
    nblk = (T + OFFSET_BLOCK - 1) // OFFSET_BLOCK
    off = _randn(g, (B, nblk, H, d), device, OFFSET_STD)
    # broadcast-add block offsets in place, chunk by chunk to bound memory
    full = T // OFFSET_BLOCK
    if full:
        noise[:, : full * OFFSET_BLOCK].view(B, full, OFFSET_BLOCK, H, d).add_(
            off[:, :full].unsqueeze(2))
    if T % OFFSET_BLOCK:
        noise[:, full * OFFSET_BLOCK:].add_(off[:, full:full + 1])
    return noise.to(torch.bfloat16)


def nsa_inputs(B: int, T: int, h_q: int, h_kv: int, d_k: int, d_v: int,
               cmp_block: int = 32, seed: int = 0, device="cpu") -> NSAInputs:
    g = _gen(seed, device)
    q = _randn(g, (B, T, h_q, d_k), device).to(torch.bfloat16)
    k = _keys(g, B, T, h_kv, d_k, device)
    v = _randn(g, (B, T, h_kv, d_v), device).to(torch.bfloat16)
    w_k = _randn(g, (cmp_block * d_k, d_k), device, 1.0 / math.sqrt(cmp_block * d_k)).to(torch.bfloat16)
    w_v = _randn(g, (cmp_block * d_v, d_v), device, 1.0 / math.sqrt(cmp_block * d_v)).to(torch.bfloat16)
    gates = torch.sigmoid(_randn(g, (B, T, h_q, 3), device)).to(torch.bfloat16)
    return NSAInputs(q, k, v, w_k, w_v, gates)


def decode_inputs(B: int, L: int, h_q: int, h_kv: int, d_k: int, d_v: int,
                  cmp_block: int = 32, seed: int = 0, device="cpu") -> DecodeInputs:
    g = _gen(seed, device)
    q = _randn(g, (B, h_q, d_k), device).to(torch.bfloat16)
    k = _keys(g, B, L, h_kv, d_k, device)
    v = _randn(g, (B, L, h_kv, d_v), device).to(torch.bfloat16)
    w_k = _randn(g, (cmp_block * d_k, d_k), device, 1.0 / math.sqrt(cmp_block * d_k)).to(torch.bfloat16)
    w_v = _randn(g, (cmp_block * d_v, d_v), device, 1.0 / math.sqrt(cmp_block * d_v)).to(torch.bfloat16)
    gates = torch.sigmoid(_randn(g, (B, h_q, 3), device)).to(torch.bfloat16)
    seqlens = torch.full((B,), L, dtype=torch.int32, device=device)
    return DecodeInputs(q, k, v, w_k, w_v, gates, seqlens)


@dataclasses.dataclass
class DsaInputs:
    q: torch.Tensor          # [B, T, H_q, d_k] bf16
    k: torch.Tensor          # [B, T, H_kv, d_k] bf16
    v: torch.Tensor          # [B, T, H_kv, d_v] bf16
    q_idx: torch.Tensor      # [B, T, H_I, d_I] bf16
    k_idx: torch.Tensor      # [B, T, d_I] bf16
    w_idx: torch.Tensor      # [B, T, H_I] bf16


def dsa_inputs(B: int, T: int, h_q: int, h_kv: int, d_k: int, d_v: int, h_i: int, d_i: int, seed: int = 0,
               device="cpu") -> DsaInputs:
    """q, k (with the 64-token key offsets), v as for NSA, then the indexer tensors: q_idx ~ N(0, 1),
    k_idx ~ N(0, 1) plus its own per-64-token offset ~ N(0, 0.5^2), w_idx ~ N(0, 1/h_i); drawn in
    that order in fp32 and rounded to bf16."""
    g = _gen(seed, device)
    q = _randn(g, (B, T, h_q, d_k), device).to(torch.bfloat16)
    k = _keys(g, B, T, h_kv, d_k, device)
    v = _randn(g, (B, T, h_kv, d_v), device).to(torch.bfloat16)
    q_idx = _randn(g, (B, T, h_i, d_i), device).to(torch.bfloat16)
    k_idx = _keys(g, B, T, 1, d_i, device)[:, :, 0].contiguous()
    w_idx = _randn(g, (B, T, h_i), device, 1.0 / math.sqrt(h_i)).to(torch.bfloat16)
    return DsaInputs(q, k, v, q_idx, k_idx, w_idx)


def phi_mlp_weights(l: int, d: int, seed: int = 0, device="cpu"):
    """Weights of phi as a two-layer MLP of hidden width d: w1 ~ N(0, 1/(l*d)) [l*d, d],
    b1 ~ N(0, 0.1^2) [d], w2 ~ N(0, 1/d) [d, d]; drawn in that order in fp32, rounded to bf16."""
    g = _gen(seed, device)
    w1 = _randn(g, (l * d, d), device, 1.0 / math.sqrt(l * d)).to(torch.bfloat16)
    b1 = _randn(g, (d,), device, 0.1).to(torch.bfloat16)
    w2 = _randn(g, (d, d), device, 1.0 / math.sqrt(d)).to(torch.bfloat16)
    return w1, b1, w2


def nsa_varlen_inputs(lengths, h_q: int, h_kv: int, d_k: int, d_v: int, cmp_block: int = 32, seed: int = 0,
                      device="cpu"):
    """A packed variable-length batch: sequence i is its own draw of nsa_inputs(1, L_i, ...)
    with seed + i (the compression weights are sequence 0's), concatenated along the tokens.
    Returns (NSAInputs with [total, ...] tensors and [l*d, d] weights, cu_seqlens int32 [B+1])."""
    xs = [nsa_inputs(1, max(int(L), 1), h_q, h_kv, d_k, d_v, cmp_block, seed + i, device)
          for i, L in enumerate(lengths)]
    cat = lambda name: torch.cat([getattr(x, name)[0, :int(L)] for x, L in zip(xs, lengths)])
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    packed = NSAInputs(cat("q"), cat("k"), cat("v"), xs[0].w_k, xs[0].w_v, cat("gates"))
    return packed, torch.tensor(cu, dtype=torch.int32, device=device)


def moba_inputs(B: int, T: int, h: int, d: int, seed: int = 0, device="cpu") -> MobaInputs:
    g = _gen(seed, device)
    q = _randn(g, (B, T, h, d), device).to(torch.bfloat16)
    k = _keys(g, B, T, h, d, device)
    v = _randn(g, (B, T, h, d), device).to(torch.bfloat16)
    return MobaInputs(q, k, v)


def one_hot_gates(B: int, T: int, h_q: int, branch: int, device="cpu") -> torch.Tensor:
    """Gates that switch on one branch (0 = compressed, 1 = selected, 2 = window)."""
    g = torch.zeros((B, T, h_q, 3), dtype=torch.bfloat16, device=device)
    g[..., branch] = 1.0
    return g


# The workloads the library is measured and checked on.
WORKLOADS = {
    "nsa_tiny": dict(B=1, T=1024, h_q=4, h_kv=1, d_k=64, d_v=64, top_k=4, window=128),
    "nsa_8k": dict(B=1, T=8192, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=16, window=512),
    "nsa_64k": dict(B=1, T=65536, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=16, window=512),
    "nsa_decode": dict(B=32, L=65536, h_q=64, h_kv=4, d_k=192, d_v=128, top_k=16, window=512),
    "moba_128k": dict(B=1, T=131072, h=32, d=128, block=512, top_k=3),
    # DSA (token-wise sparse attention): 4 indexer heads of 64 dims, 2048 tokens per query
    "dsa_8k": dict(B=1, T=8192, h_q=64, h_kv=4, d_k=192, d_v=128, h_i=4, d_i=64, top_k=2048),
    # a packed batch of 8 sequences of different lengths, 65536 tokens in all
    "nsa_varlen": dict(lengths=(16384, 12288, 9000, 8192, 7000, 5000, 4096, 3576), h_q=64, h_kv=4, d_k=192,
                       d_v=128, top_k=16, window=512),
}
