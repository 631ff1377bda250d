"""Seeded synthetic workloads for DCA prefill and decode.

Shared by the tests, the benchmark and the oracle comparisons.  This module
holds no attention or RoPE arithmetic: it only draws random numbers.

Recipe (every config, seed 0 unless stated):
  * one ``torch.Generator`` on the requested device, seeded once;
  * prefill: Q [B, L, Hq, D], then K [B, L, Hkv, D], then V [B, L, Hkv, D],
    each drawn as float32 N(0, 1) and rounded to bf16 (round to nearest even);
  * "K x2 on 1% of positions": n = floor(frac * L) token positions from a
    ``randperm(L)`` drawn after V; K is doubled at those positions for every
    batch entry and kv head (exact in bf16);
  * packed variable-length batch: lengths [B] uniform integers in
    [len_lo, len_hi] drawn first (or given), cu_seqlens their running sums
    from 0, then Q [T, Hq, D], K [T, Hkv, D], V [T, Hkv, D] as for prefill;
  * decode: t [B] uniform integers in [t_lo, t_hi) drawn first, then q
    [B, Hq, D], then the K cache entry by entry (K[b] = [Tcap, Hkv, D] for
    b = 0 .. B-1), then the V cache the same way.  The K cache stands for keys
    already rotated at j mod s: a rotation of i.i.d. N(0, 1) pairs is again
    i.i.d. N(0, 1), so the draw itself is a valid pre-rotated cache.

The same recipe on another device gives other numbers (CPU and CUDA
generators differ); tests that compare against the oracle draw on the CPU and
copy to the GPU.
"""

from __future__ import annotations

import torch

# Llama-2 attention shapes at the context lengths of the DCA evaluation
# (7B: 32 heads; 70B: 64 query heads over 8 kv heads), pretraining length 4096.
CONFIGS = {
    "tiny": dict(kind="prefill", B=1, L=1024, Hq=1, Hkv=1, D=64, c=256, s=192,
                 base=10000.0, k_boost_frac=0.0),
    "llama2_7b_16k": dict(kind="prefill", B=1, L=16384, Hq=32, Hkv=32, D=128,
                          c=4096, s=3072, base=10000.0, k_boost_frac=0.0),
    "llama2_70b_32k": dict(kind="prefill", B=1, L=32768, Hq=64, Hkv=8, D=128,
                           c=4096, s=3072, base=10000.0, k_boost_frac=0.01),
    "prefill_100k": dict(kind="prefill", B=1, L=100000, Hq=64, Hkv=8, D=128,
                         c=4096, s=3072, base=10000.0, k_boost_frac=0.0),
    "decode_b16": dict(kind="decode", B=16, Hq=64, Hkv=8, D=128, Tcap=65536,
                       c=4096, s=3072, base=10000.0, t_lo=32768, t_hi=65536),
    # packed batch of prompts of mixed length (serving-style prefill)
    "varlen_7b_mix": dict(kind="varlen", B=8, Hq=32, Hkv=32, D=128, c=4096, s=3072,
                          base=10000.0, len_lo=512, len_hi=16384),
}


def _normal_bf16(shape, gen, device):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_prefill_inputs(cfg: dict, device="cpu", seed: int = 0):
    """Return (Q, K, V) bf16 tensors on ``device`` following the recipe."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, L, Hq, Hkv, D = cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"]
    Q = _normal_bf16((B, L, Hq, D), gen, device)
    K = _normal_bf16((B, L, Hkv, D), gen, device)
    V = _normal_bf16((B, L, Hkv, D), gen, device)
    frac = cfg.get("k_boost_frac", 0.0)
    if frac:
        n = int(frac * L)
        pos = torch.randperm(L, generator=gen, device=device)[:n]
        K[:, pos] = K[:, pos] * 2
    return Q, K, V


def make_varlen_inputs(cfg: dict, device="cpu", seed: int = 0, lens=None):
    """Return (Q [T,Hq,D], K, V [T,Hkv,D] bf16 on ``device``, cu_seqlens int32
    [B+1] on the CPU, lens list) for a packed batch of mixed-length prompts."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    if lens is None:
        lens = torch.randint(cfg["len_lo"], cfg["len_hi"] + 1, (cfg["B"],), generator=gen,
                             device=device, dtype=torch.int64).tolist()
    lens = [int(n) for n in lens]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    Hq, Hkv, D = cfg["Hq"], cfg["Hkv"], cfg["D"]
    Q = _normal_bf16((T, Hq, D), gen, device)
    K = _normal_bf16((T, Hkv, D), gen, device)
    V = _normal_bf16((T, Hkv, D), gen, device)
    return Q, K, V, cu, lens


def boosted_positions(cfg: dict, seed: int = 0):
    """Token positions whose K was doubled (replays the draws on the CPU)."""
    frac = cfg.get("k_boost_frac", 0.0)
    if not frac:
        return torch.empty(0, dtype=torch.int64)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    B, L, Hq, Hkv, D = cfg["B"], cfg["L"], cfg["Hq"], cfg["Hkv"], cfg["D"]
    for shape in ((B, L, Hq, D), (B, L, Hkv, D), (B, L, Hkv, D)):
        torch.randn(shape, generator=gen, dtype=torch.float32)
    return torch.randperm(L, generator=gen)[: int(frac * L)]


def make_decode_inputs(cfg: dict, device="cpu", seed: int = 0):
    """Return (t int32 [B], q [B,Hq,D], Kcache, Vcache [B,Tcap,Hkv,D]) bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, Hq, Hkv, D, T = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["Tcap"]
    t = torch.randint(cfg["t_lo"], cfg["t_hi"], (B,), generator=gen,
                      device=device, dtype=torch.int64).to(torch.int32)
    q = _normal_bf16((B, Hq, D), gen, device)
    Kc = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=device)
    Vc = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=device)
    for b in range(B):
        Kc[b] = _normal_bf16((T, Hkv, D), gen, device)
    for b in range(B):
        Vc[b] = _normal_bf16((T, Hkv, D), gen, device)
    return t, q, Kc, Vc


def scaled(cfg: dict, **over) -> dict:
    """A copy of ``cfg`` with some sizes replaced (smaller parity cases)."""
    out = dict(cfg)
    out.update(over)
    return out


def prefill_flops(cfg: dict) -> float:
    """Algorithmic FLOPs of causal attention: 4 * D * Hq * B * L(L+1)/2."""
    L = cfg["L"]
    return 4.0 * cfg["D"] * cfg["Hq"] * cfg["B"] * L * (L + 1) / 2


def varlen_flops(lens, Hq: int, D: int) -> float:
    """Algorithmic FLOPs of a packed batch: causal attention per sequence."""
    return sum(4.0 * D * Hq * n * (n + 1) / 2 for n in lens)


def varlen_chunk_flops(t0, lens, Hq: int, D: int) -> float:
    """Algorithmic FLOPs of packed chunks over caches: row r of sequence b
    attends t0[b] + r + 1 keys."""
    return sum(4.0 * D * Hq * (n * a + n * (n + 1) / 2) for a, n in zip(t0, lens))


def decode_bytes(cfg: dict, t) -> float:
    """Algorithmic bytes of one decode step.

    K and V of the valid prefix (t_b + 1 keys) read once per kv head, bf16,
    plus the bf16 query in and bf16 output / fp32 LSE out.
    """
    D, Hkv, Hq, B = cfg["D"], cfg["Hkv"], cfg["Hq"], cfg["B"]
    kv = sum(int(x) + 1 for x in t) * Hkv * D * 2 * 2
    return float(kv + B * Hq * D * 2 * 2 + B * Hq * 4)
