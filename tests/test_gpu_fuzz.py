"""Seeded random shapes through the prefill entry points, against the oracle.

Each case draws batch, length, heads (GQA groups 1, 2 or 8), head dimension,
pretraining length c and chunk size s (any 1 <= s <= c, with a third of the
cases on multiples of 256 so the two-tile kernel is reached too) from a fixed
seed.  dca_attn_prefill is compared with the fp64 oracle on the rows that
stress the index rule plus random rows; the same sequences cut to random
lengths and packed go through dca_attn_prefill_varlen and must give, bit for
bit, what dca_attn_prefill gives on each sequence alone.
"""

import numpy as np
import pytest
import torch

import long_context_attention_dca_b200 as dca
from oracle import dca_oracle as orc
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

N_CASES = 40


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_attention_dca_b200 import build
    build.build()
    dca.lib()
    yield
    dca.dca_sync_status()


def _case(k):
    rng = np.random.default_rng(1000 + k)
    D = int(rng.choice([64, 128]))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 8]))
    while Hkv * G > 16:
        G //= 2
    if k % 3 == 0:
        s = int(rng.choice([256, 512]))
        c = s + int(rng.integers(0, 400))
    else:
        c = int(rng.integers(8, 700))
        s = int(rng.integers(1, c + 1))
    B = int(rng.integers(1, 3))
    L = int(rng.integers(1, 900))
    return dict(B=B, L=L, Hq=Hkv * G, Hkv=Hkv, D=D, s=s, c=c, seed=2000 + k)


def _inputs(cs):
    gen = torch.Generator().manual_seed(cs["seed"])
    B, L, Hq, Hkv, D = cs["B"], cs["L"], cs["Hq"], cs["Hkv"], cs["D"]
    Q = torch.randn(B, L, Hq, D, generator=gen).to(torch.bfloat16)
    K = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    V = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    return Q, K, V


@pytest.mark.parametrize("k", range(N_CASES))
def test_random_shape_prefill_matches_oracle(k):
    cs = _case(k)
    Q, K, V = _inputs(cs)
    s, c = cs["s"], cs["c"]
    O, LSE = dca.dca_attn_prefill(Q.cuda(), K.cuda(), V.cuda(), s, c)
    dca.dca_sync_status()
    rows = pu.sample_rows(cs["L"], s, c, n_random=24, seed=k)
    heads = pu.sample_heads(cs["Hq"], cs["Hkv"])
    ref = orc.dca_prefill_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V), s, c,
                               rows=rows, heads=heads)
    mx, mean, lse = pu.compare_rows(O.cpu(), LSE.cpu(), ref)
    print(f"{cs}: O max {mx:.3e} mean {mean:.3e} LSE rel {lse:.3e}")
    pu.assert_close(mx, mean, lse, str(cs))


@pytest.mark.parametrize("k", range(N_CASES))
def test_random_shape_varlen_equals_per_sequence(k):
    cs = _case(k)
    Q, K, V = _inputs(cs)
    s, c = cs["s"], cs["c"]
    rng = np.random.default_rng(3000 + k)
    lens = [int(rng.integers(0, cs["L"] + 1)) for _ in range(cs["B"])] + [cs["L"]]
    Qp = torch.cat([Q[b % cs["B"], :n] for b, n in enumerate(lens)])
    Kp = torch.cat([K[b % cs["B"], :n] for b, n in enumerate(lens)])
    Vp = torch.cat([V[b % cs["B"], :n] for b, n in enumerate(lens)])
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    O, LSE = dca.dca_attn_prefill_varlen(Qp.cuda(), Kp.cuda(), Vp.cuda(), cu.cuda(), max(lens),
                                         s, c)
    dca.dca_sync_status()
    O, LSE = O.cpu(), LSE.cpu()
    for b, n in enumerate(lens):
        if n == 0:
            continue
        a = int(cu[b])
        src = b % cs["B"]
        Ob, Lb = dca.dca_attn_prefill(Q[src:src + 1, :n].contiguous().cuda(),
                                      K[src:src + 1, :n].contiguous().cuda(),
                                      V[src:src + 1, :n].contiguous().cuda(), s, c)
        dca.dca_sync_status()
        assert torch.equal(O[a:a + n], Ob[0].cpu()), (cs, lens, b)
        assert torch.equal(LSE[:, a:a + n], Lb[0].cpu()), (cs, lens, b)


@pytest.mark.parametrize("k", range(N_CASES // 2))
def test_random_shape_varlen_chunk_matches_oracle(k):
    # the same shapes as packed chunks over caches: random cached lengths and
    # chunk lengths (some empty), random cache contents standing for rotated
    # keys; every row against the oracle
    cs = _case(k)
    rng = np.random.default_rng(4000 + k)
    B = int(rng.integers(1, 5))
    t0 = [int(rng.integers(0, 600)) for _ in range(B)]
    lens = [int(rng.integers(0, 300)) for _ in range(B)]
    lens[-1] = max(lens[-1], 1)
    Hq, Hkv, D, s, c = cs["Hq"], cs["Hkv"], cs["D"], cs["s"], cs["c"]
    gen = torch.Generator().manual_seed(5000 + k)
    T = sum(lens)
    Tcap = max(a + n for a, n in zip(t0, lens)) + int(rng.integers(0, 200))
    Q = torch.randn(T, Hq, D, generator=gen).to(torch.bfloat16)
    K = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    V = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    Kc = torch.randn(B, Tcap, Hkv, D, generator=gen).to(torch.bfloat16)
    Vc = torch.randn(B, Tcap, Hkv, D, generator=gen).to(torch.bfloat16)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    max_kv = max(a + n for a, n in zip(t0, lens))
    O, LSE = dca.dca_attn_prefill_varlen_chunk(
        Q.cuda(), K.cuda(), V.cuda(), Kc.cuda(), Vc.cuda(), cu.cuda(),
        torch.tensor(t0, dtype=torch.int32, device="cuda"), max(lens), max_kv, s, c)
    dca.dca_sync_status()
    O, LSE = O.cpu(), LSE.cpu()
    ref = orc.dca_prefill_varlen_chunk_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                            cu.tolist(), t0, pu.F64View(Kc), pu.F64View(Vc),
                                            s, c)
    keys = sorted(ref)
    o_ref = np.stack([ref[key][0] for key in keys])
    l_ref = np.array([ref[key][1] for key in keys])
    o_got = np.stack([O[t, h].double().numpy() for h, t in keys])
    l_got = np.array([float(LSE[h, t]) for h, t in keys])
    err = np.abs(o_got - o_ref)
    lse = float(np.max(np.abs(l_got - l_ref) / np.maximum(np.abs(l_ref), 1.0)))
    print(f"{cs} t0={t0} lens={lens}: O max {err.max():.3e} mean {err.mean():.3e} "
          f"LSE rel {lse:.3e}")
    pu.assert_close(float(err.max()), float(err.mean()), lse, f"{cs} t0={t0} lens={lens}")
