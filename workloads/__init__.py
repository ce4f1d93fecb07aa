"""Seeded synthetic inputs for the Reduced Matrix Multiplication workloads.

This module draws random inputs with the shapes and value distributions of the
five RMM workloads and nothing else: it computes no column score, no
selection and no product.  Both the CUDA path's tests and the CPU oracle's
tests take their inputs from here.  Where a test needs a safety gap between
the scores on either side of the selection boundary, it measures the scores
with the oracle and passes per-column gains back in (``col_gain``); the gains
are applied before the final rounding to the storage dtype.

Distributions ("N(mu, sigma)" = mean and standard deviation; LogN(0,1) =
exp(N(0,1))):
  linear_small   fp32 A n x d = N(0,1) * LogN(0,1) per column; B d x m = N(0, 0.02)
  mlp_up         bf16 A n x 4096 = N(0,1) * LogN(0,1) per channel, 1% of the
                 channels (seeded choice) x20; B 4096 x 14336 = N(0, 0.02)
  mlp_down       bf16 A n x 14336 = SiLU(N(0,1)); B 14336 x 4096 = N(0, 0.02)
  attn_qk        bf16 Q [H][n][d_h], K [H_kv][n][d_h] = N(0,1) * LogN(0,1) per
                 (head, feature), a separate draw per head
  attn_pv        bf16 P [H][n][n] = row softmax of causal N(0,2) logits;
                 V [H_kv][n][d_v] = N(0,1)
  linear_70b     bf16 B in {8192x28672, 28672x8192, 8192x10240} = N(0, 0.014);
                 A as mlp_up (d = 8192) or as mlp_down (d = 28672)
  quantize_e4m3  per-tensor 8-bit E4M3 codes (scale = amax / 448) of any of the
                 above, for the low-bit form
  attn_decode    one decode step per sequence: q [B*H][n][d_h] and the K cache
                 [B*H_kv][t][d_h] as attn_qk; V cache [B*H_kv][t][d_v] = N(0,1);
                 P [B*H][n][t] = row softmax of N(0,2) logits (as attn_pv),
                 each the sum of a draw shared by the query heads of one KV
                 head and one of its own (correlation 0.5)
These stand in for the Llama-family activations and weights the RMM paper
evaluates on (none of which are available here).
"""
from __future__ import annotations

import math

import torch

__all__ = [
    "gen", "linear_small", "mlp_up", "mlp_down", "attn_qk", "attn_pv", "attn_decode", "linear_70b",
    "duplicate_columns", "quantize_e4m3", "LLAMA8B_MLP", "LLAMA70B_LINEAR",
]

LLAMA8B_MLP = {"up": (4096, 14336), "down": (14336, 4096)}
LLAMA70B_LINEAR = {"up": (8192, 28672), "down": (28672, 8192), "qkv": (8192, 10240)}


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _normal(shape, g, device, std=1.0):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _apply_gain(x: torch.Tensor, col_gain) -> torch.Tensor:
    if col_gain is None:
        return x
    gain = torch.as_tensor(col_gain, dtype=torch.float64).to(x.device)
    return (x.double() * gain).float()


def linear_small(seed: int, n: int = 64, d: int = 256, m: int = 256, col_gain=None,
                 device="cpu"):
    """fp32 A (n x d) and B (d x m): the tiny oracle-scale linear workload."""
    g = gen(seed, device)
    scale = torch.exp(_normal((d,), g, device))
    A = _normal((n, d), g, device) * scale
    B = _normal((d, m), g, device, 0.02)
    return _apply_gain(A, col_gain).contiguous(), B.contiguous()


def _outlier_activations(g, n, d, device):
    scale = torch.exp(_normal((d,), g, device))
    n_out = max(1, round(0.01 * d))
    idx = torch.randperm(d, generator=g, device=device)[:n_out]
    scale[idx] *= 20.0
    return _normal((n, d), g, device) * scale


def _silu_activations(g, n, d, device):
    z = _normal((n, d), g, device)
    return z * torch.sigmoid(z)


def mlp_up(seed: int, n: int, d: int = 4096, m: int = 14336, col_gain=None, device="cpu",
           dtype=torch.bfloat16):
    """Up/gate-projection input: outlier-channel activations and a N(0,0.02) weight."""
    g = gen(seed, device)
    A = _outlier_activations(g, n, d, device)
    B = _normal((d, m), g, device, 0.02)
    return _apply_gain(A, col_gain).to(dtype).contiguous(), B.to(dtype).contiguous()


def mlp_down(seed: int, n: int, d: int = 14336, m: int = 4096, col_gain=None, device="cpu",
             dtype=torch.bfloat16):
    """Down-projection input: SiLU(N(0,1)) activations and a N(0,0.02) weight."""
    g = gen(seed, device)
    A = _silu_activations(g, n, d, device)
    B = _normal((d, m), g, device, 0.02)
    return _apply_gain(A, col_gain).to(dtype).contiguous(), B.to(dtype).contiguous()


def linear_70b(seed: int, n: int, shape: str, col_gain=None, device="cpu",
               dtype=torch.bfloat16):
    """Llama-3-70B-shaped projection: shape in {"up", "down", "qkv"}."""
    d, m = LLAMA70B_LINEAR[shape]
    g = gen(seed, device)
    if shape == "down":
        A = _silu_activations(g, n, d, device)
    else:
        A = _outlier_activations(g, n, d, device)
    B = _normal((d, m), g, device, 0.014)
    return _apply_gain(A, col_gain).to(dtype).contiguous(), B.to(dtype).contiguous()


def attn_qk(seed: int, n: int, heads: int = 32, kv_heads: int = 8, head_dim: int = 128,
            col_gain=None, device="cpu", dtype=torch.bfloat16):
    """Q [heads][n][head_dim] and K [kv_heads][n][head_dim]; col_gain is [heads][head_dim]."""
    g = gen(seed, device)
    qs = torch.exp(_normal((heads, 1, head_dim), g, device))
    Q = _normal((heads, n, head_dim), g, device) * qs
    ks = torch.exp(_normal((kv_heads, 1, head_dim), g, device))
    K = _normal((kv_heads, n, head_dim), g, device) * ks
    if col_gain is not None:
        gain = torch.as_tensor(col_gain, dtype=torch.float64).to(device)
        Q = (Q.double() * gain[:, None, :]).float()
    return Q.to(dtype).contiguous(), K.to(dtype).contiguous()


def attn_pv(seed: int, n: int, heads: int = 32, kv_heads: int = 8, v_dim: int = 128,
            col_gain=None, device="cpu", dtype=torch.bfloat16):
    """P [heads][n][n] (row softmax of causal N(0,2) logits, built one head at a
    time in fp32) and V [kv_heads][n][v_dim]; col_gain is [heads][n]."""
    g = gen(seed, device)
    P = torch.empty((heads, n, n), dtype=dtype, device=device)
    causal = torch.ones((n, n), dtype=torch.bool, device=device).triu_(1)
    for h in range(heads):
        logits = _normal((n, n), g, device, 2.0)
        logits.masked_fill_(causal, -math.inf)
        p = torch.softmax(logits, dim=-1)
        if col_gain is not None:
            gain = torch.as_tensor(col_gain[h], dtype=torch.float64).to(device)
            p = (p.double() * gain).float()
        P[h] = p.to(dtype)
        del logits, p
    V = _normal((kv_heads, n, v_dim), g, device)
    return P, V.to(dtype).contiguous()


def attn_decode(seed: int, t: int, batch: int = 1, n: int = 1, heads: int = 32, kv_heads: int = 8,
                head_dim: int = 128, v_dim: int = 128, q_gain=None, p_gain=None, device="cpu",
                dtype=torch.bfloat16):
    """One decode step of `batch` sequences with t cached tokens each (query
    heads of sequence b are b*heads .. b*heads + heads - 1, their KV heads
    b*kv_heads ..).  Returns (q, K, V, P).  q_gain [batch*heads][head_dim]
    scales q; p_gain [batch*heads][t] scales P after the softmax (both before
    the final rounding)."""
    g = gen(seed, device)
    H, Hkv = batch * heads, batch * kv_heads
    qs = torch.exp(_normal((H, 1, head_dim), g, device))
    q = _normal((H, n, head_dim), g, device) * qs
    ks = torch.exp(_normal((Hkv, 1, head_dim), g, device))
    K = _normal((Hkv, t, head_dim), g, device) * ks
    V = _normal((Hkv, t, v_dim), g, device)
    group = heads // kv_heads
    shared = _normal((Hkv, n, t), g, device).repeat_interleave(group, dim=0)
    logits = 2.0 * math.sqrt(0.5) * (shared + _normal((H, n, t), g, device))
    del shared
    P = torch.softmax(logits, dim=-1)
    del logits
    if q_gain is not None:
        gain = torch.as_tensor(q_gain, dtype=torch.float64).to(device)
        q = (q.double() * gain[:, None, :]).float()
    if p_gain is not None:
        gain = torch.as_tensor(p_gain, dtype=torch.float64).to(device)
        P = (P.double() * gain[:, None, :]).float()
    return q.to(dtype).contiguous(), K.to(dtype).contiguous(), V.to(dtype).contiguous(), P.to(dtype).contiguous()


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor 8-bit E4M3 codes of x and their scale: scale = amax / 448
    (the largest E4M3 magnitude), codes = round-to-nearest(x / scale) as
    torch's float8_e4m3fn conversion gives them.  Returns (codes, scale);
    x ~ codes * scale.  Input preparation for the low-bit form only."""
    xf = x.float()
    amax = float(xf.abs().max())
    scale = amax / 448.0 if amax > 0 else 1.0
    return (xf / scale).to(torch.float8_e4m3fn).contiguous(), scale


def duplicate_columns(A: torch.Tensor, pairs) -> torch.Tensor:
    """Copy column src into column dst for each (src, dst): an exact-tie input."""
    A = A.clone()
    for src, dst in pairs:
        A[..., dst] = A[..., src]
    return A
