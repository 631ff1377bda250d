"""Host checks of the seeded workload generators and of the algorithmic work
counts the benchmark divides by (CPU only)."""

import numpy as np
import torch

from long_context_attention_dca_b200 import workloads as W
from oracle import dca_oracle as orc


def test_prefill_inputs_follow_the_recipe():
    cfg = W.scaled(W.CONFIGS["llama2_70b_32k"], L=300, Hq=4, Hkv=2, D=64)
    Q, K, V = W.make_prefill_inputs(cfg, seed=3)
    Q2, K2, V2 = W.make_prefill_inputs(cfg, seed=3)
    assert Q.dtype == K.dtype == V.dtype == torch.bfloat16
    assert Q.shape == (1, 300, 4, 64) and K.shape == V.shape == (1, 300, 2, 64)
    assert torch.equal(Q, Q2) and torch.equal(K, K2) and torch.equal(V, V2)
    # K doubled at floor(0.01 L) = 3 seeded positions, the rest as drawn
    pos = W.boosted_positions(cfg, seed=3)
    assert len(pos) == 3
    plain = W.make_prefill_inputs(dict(cfg, k_boost_frac=0.0), seed=3)[1]
    keep = [i for i in range(300) if i not in set(pos.tolist())]
    assert torch.equal(K[:, keep], plain[:, keep])
    assert torch.equal(K[:, pos], (plain[:, pos].float() * 2).to(torch.bfloat16))


def test_varlen_inputs_pack_their_lengths():
    cfg = W.CONFIGS["varlen_7b_mix"]
    small = dict(cfg, Hq=2, Hkv=2, D=64, B=5, len_lo=3, len_hi=40)
    Q, K, V, cu, lens = W.make_varlen_inputs(small, seed=1)
    assert len(lens) == 5 and all(3 <= n <= 40 for n in lens)
    assert cu.dtype == torch.int32 and cu[0] == 0 and (cu[1:] - cu[:-1]).tolist() == lens
    assert Q.shape == (sum(lens), 2, 64) and K.shape == V.shape == (sum(lens), 2, 64)
    _, _, _, cu2, lens2 = W.make_varlen_inputs(small, seed=1, lens=[0, 7, 0])
    assert lens2 == [0, 7, 0] and cu2.tolist() == [0, 0, 7, 7]


def _causal_pairs(L):
    _, _, piece = orc.index_map(L, 3, 5)
    return int((piece >= 0).sum())


def test_work_counts_match_brute_force():
    # prefill FLOPs = 4 D Hq B x (causal pairs), pairs counted from the
    # oracle's index map
    for L in (1, 7, 33):
        cfg = dict(B=2, L=L, Hq=3, D=64)
        assert W.prefill_flops(cfg) == 4 * 64 * 3 * 2 * _causal_pairs(L)
    lens = [1, 7, 0, 33]
    assert W.varlen_flops(lens, 3, 64) == sum(4 * 64 * 3 * _causal_pairs(n) for n in lens if n)
    # a chunk of n rows at offset t0: row r attends t0 + r + 1 keys
    t0 = [0, 5, 12, 100]
    want = sum(4 * 64 * 3 * sum(a + r + 1 for r in range(n)) for a, n in zip(t0, lens))
    assert W.varlen_chunk_flops(t0, lens, 3, 64) == want
    # decode bytes: K and V of keys 0 .. t per sequence and kv head, plus q, O, LSE
    cfg = dict(B=2, Hq=8, Hkv=2, D=64)
    t = np.array([0, 99])
    assert W.decode_bytes(cfg, t) == (1 + 100) * 2 * 64 * 2 * 2 + 2 * 8 * 64 * 2 * 2 + 2 * 8 * 4
